/*
 * ssu_oracle.c -- plain, slow float64 CPU oracle for the Mamba selective state update.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg call this code; the product path never does. It shares no code,
 * header or constant with the CUDA library.
 *
 * Source of the method: "Selective State Update" page of the TensorRT-Edge-LLM C++ API
 * (mamba_ssm::invokeSelectiveStateUpdate, invokeSelectiveStateUpdatePrefill,
 * struct MambaReplayLayerInfo, invokeMambaStateClear), the padding contract of the
 * FlashInfer page "flashinfer.gdn_fused_decode_step" (parameter state_indices), and the
 * "Recurrent State Manager" page (clearSlot, copySlotFrom).
 *
 * Per active row b and head h, one token does
 *     dt_eff    = softplus(dt + dt_bias)  (or dt + dt_bias when softplus is off)
 *     new_state = state * exp(A * dt_eff) + B * dt_eff * x
 *     out       = sum_n new_state[n] * C[n] + D * x,   then out *= silu(z) if z is given
 * Everything is computed in double. Inputs are decoded exactly from their storage type;
 * the pool is read in its storage type and the final state is rounded once (to nearest,
 * ties to even) when it is stored back. Outputs are returned unrounded, in double.
 * The (row, head) units of a call are independent (each owns its state block, outputs
 * and stash entries), so they run in parallel on OpenMP threads; the arithmetic of one
 * unit is the same sequential loop whatever the thread count.
 *
 * Readings taken where the pages leave a point open:
 *   - head h uses group g = h / (H / G) (contiguous blocks of heads per group);
 *   - dt_bias is added whenever it is given, with or without softplus;
 *   - the replay stash holds DA = exp(A * dt_eff) (the decay factor), DT = dt_eff,
 *     U = x and B, all fp32, because the replay call receives no A, dt_bias or softplus;
 *   - positions t >= contextLengths[b] are neither read nor written; a row whose length
 *     is 0 is left untouched;
 *   - a padding row (stateIndices[b] < 0) reads and writes no state; its outputs are 0
 *     (all T positions in prefill); the replay writes nothing for it;
 *   - an index >= P, a length > T or a negative length is undefined on the pages; here
 *     the row is skipped (index) or the length clamped, and a bit is set in err_flags:
 *     1 = index >= P, 2 = acceptedLengths > T, 4 = contextLengths > T, 8 = negative length,
 *     64 = malformed tree input (see the tree verify below).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* storage types understood by the oracle */
enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2, OR_F64 = 3 };

/* ---------------- exact decoding of the storage formats ---------------- */

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double oracle_f16_to_double(uint16_t h)
{
    int sign = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);              /* zero or subnormal */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);  /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ---------------- rounding to nearest, ties to even ---------------- */

/* Round v to a binary format with p significand bits (implicit bit included),
 * minimum normal exponent emin and maximum exponent emax. */
static double round_to_format(double v, int p, int emin, int emax)
{
    if (isnan(v) || isinf(v) || v == 0.0)
        return v;
    double a = fabs(v);
    int E;
    frexp(a, &E);           /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;          /* a in [2^e, 2^(e+1)) */
    if (e < emin)
        e = emin;           /* subnormal range: fixed quantum */
    double q = ldexp(1.0, e - (p - 1));
    double r = nearbyint(a / q) * q;   /* default mode: to nearest, ties to even */
    double maxfin = ldexp(2.0 - ldexp(1.0, -(p - 1)), emax);
    if (r > maxfin)
        r = INFINITY;
    return copysign(r, v);
}

uint16_t oracle_double_to_f16(double v)
{
    if (isnan(v))
        return 0x7e00;
    double r = round_to_format(v, 11, -14, 15);
    uint16_t sign = signbit(r) ? 0x8000 : 0;
    double a = fabs(r);
    if (isinf(a))
        return sign | 0x7c00;
    if (a < ldexp(1.0, -14))                 /* subnormal: a = m * 2^-24 exactly */
        return sign | (uint16_t)(a / ldexp(1.0, -24));
    int E;
    double f = frexp(a, &E);                 /* a = (2f) * 2^(E-1), 2f in [1, 2) */
    uint16_t frac = (uint16_t)((2.0 * f - 1.0) * 1024.0);
    return sign | (uint16_t)((E - 1 + 15) << 10) | frac;
}

uint16_t oracle_double_to_bf16(double v)
{
    if (isnan(v))
        return 0x7fc0;
    /* every bfloat16 value is exactly a binary32, whose upper half is the encoding */
    float f = (float)round_to_format(v, 8, -126, 127);
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(bits >> 16);
}

/* ---------------- typed element access ---------------- */

static double load(const void *p, int dt, int64_t i)
{
    switch (dt) {
    case OR_F32: return (double)((const float *)p)[i];
    case OR_F16: return oracle_f16_to_double(((const uint16_t *)p)[i]);
    case OR_BF16: return oracle_bf16_to_double(((const uint16_t *)p)[i]);
    default: return ((const double *)p)[i];
    }
}

static void store(void *p, int dt, int64_t i, double v)
{
    switch (dt) {
    case OR_F32: ((float *)p)[i] = (float)v; break;   /* C conversion: to nearest even */
    case OR_F16: ((uint16_t *)p)[i] = oracle_double_to_f16(v); break;
    case OR_BF16: ((uint16_t *)p)[i] = oracle_double_to_bf16(v); break;
    default: ((double *)p)[i] = v; break;
    }
}

static int valid_dtype(int dt) { return dt >= OR_F32 && dt <= OR_F64; }

/* ---------------- scalar helpers ---------------- */

/* softplus(v) = log(1 + e^v), written so that neither branch overflows */
static double softplus(double v)
{
    return v > 0.0 ? v + log1p(exp(-v)) : log1p(exp(v));
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* dt after the optional bias and the optional softplus */
static double effective_dt(double dt, const float *dt_bias, int h, int dt_softplus)
{
    double v = dt + (dt_bias ? (double)dt_bias[h] : 0.0);
    return dt_softplus ? softplus(v) : v;
}

/* Resolve row b to a pool slot. Returns the slot, -1 for a padding row, or -2 when
 * the index is out of range (flag bit 1 set). */
static int64_t resolve_slot(const int32_t *state_indices, int32_t b, int32_t P,
                            int32_t *err)
{
    int64_t s = state_indices ? state_indices[b] : b;
    if (s < 0)
        return -1;
    if (s >= P) {
        *err |= 1;
        return -2;
    }
    return s;
}

static int check_common(int32_t batch, int32_t active, int32_t H, int32_t G,
                        int32_t Dm, int32_t N, int64_t slot_stride)
{
    if (batch < 0 || active < 0 || active > batch)
        return 2;
    if (H <= 0 || G <= 0 || Dm <= 0 || N <= 0 || H % G != 0)
        return 2;
    if (slot_stride < (int64_t)H * Dm * N)
        return 2;
    return 0;
}

/* ---------------- decode (seq_len == 1) ----------------
 * Selective State Update page, mamba_ssm::invokeSelectiveStateUpdate:
 * x [batch,H,Dm], A [H], B/C [batch,G,N], dt [batch,H], dt_bias/D [H], z like x,
 * state pool [P,H,Dm,N] updated in place through stateIndices, output [batch,H,Dm]. */
int oracle_decode(const void *x, int x_dt, const float *A,
                  const void *B, const void *C, int bc_dt,
                  const float *dt, const float *dt_bias, const float *D, const void *z,
                  void *pool, int state_dt, int64_t slot_stride, int32_t P,
                  double *out, const int32_t *state_indices,
                  int32_t batch, int32_t active, int32_t H, int32_t G, int32_t Dm,
                  int32_t N, int dt_softplus, int32_t *err_flags)
{
    if (!x || !A || !B || !C || !dt || !pool || !out)
        return 1;
    if (!valid_dtype(x_dt) || !valid_dtype(bc_dt) || !valid_dtype(state_dt))
        return 3;
    if (check_common(batch, active, H, G, Dm, N, slot_stride))
        return 2;
    int32_t err = 0;
    const int heads_per_group = H / G;
    const int64_t units = (int64_t)active * H;
    /* every (row, head) unit owns its state block and its output rows */
#pragma omp parallel for schedule(dynamic, 1) reduction(|:err)
    for (int64_t u = 0; u < units; ++u) {
        const int32_t b = (int32_t)(u / H);
        const int h = (int)(u % H);
        int64_t s = resolve_slot(state_indices, b, P, &err);
        if (s == -1) {                       /* padding row: output zero, no state */
            for (int d = 0; d < Dm; ++d)
                out[((int64_t)b * H + h) * Dm + d] = 0.0;
            continue;
        }
        if (s < 0)
            continue;
        double *snew = malloc(sizeof(double) * (size_t)N);
        int g = h / heads_per_group;
        double dte = effective_dt(dt[(int64_t)b * H + h], dt_bias, h, dt_softplus);
        double decay = exp((double)A[h] * dte);
        for (int d = 0; d < Dm; ++d) {
            int64_t xi = ((int64_t)b * H + h) * Dm + d;
            double xv = load(x, x_dt, xi);
            double y = 0.0;
            for (int n = 0; n < N; ++n) {
                int64_t si = s * slot_stride + ((int64_t)h * Dm + d) * N + n;
                int64_t bi = ((int64_t)b * G + g) * N + n;
                snew[n] = load(pool, state_dt, si) * decay
                          + load(B, bc_dt, bi) * dte * xv;
                y += snew[n] * load(C, bc_dt, bi);
            }
            for (int n = 0; n < N; ++n)
                store(pool, state_dt, s * slot_stride + ((int64_t)h * Dm + d) * N + n,
                      snew[n]);
            if (D)
                y += (double)D[h] * xv;
            if (z)
                y *= silu(load(z, x_dt, xi));
            out[xi] = y;
        }
        free(snew);
    }
    if (err_flags)
        *err_flags |= err;
    return 0;
}

/* ---------------- prefill (seq_len > 1) ----------------
 * Selective State Update page, mamba_ssm::invokeSelectiveStateUpdatePrefill:
 * x, z, out [batch,T,H,Dm]; B, C [batch,T,G,N]; dt [batch,T,H]; all T tokens in one
 * call, with optional contextLengths. With the replay stash (DA, U, Bst, DT, all fp32:
 * [batch,T,H], [batch,T,H,Dm], [batch,T,G,N], [batch,T,H]) the committed state is
 * read only and the per-token replay inputs are written instead. Without the stash
 * the state after L_b tokens is stored back once. The state stays in double across
 * the tokens (no rounding between tokens). */
int oracle_prefill(const void *x, int x_dt, const float *A,
                   const void *B, const void *C, int bc_dt,
                   const float *dt, const float *dt_bias, const float *D, const void *z,
                   void *pool, int state_dt, int64_t slot_stride, int32_t P,
                   double *out, const int32_t *state_indices,
                   const int32_t *context_lengths,
                   float *st_DA, float *st_U, float *st_B, float *st_DT,
                   int32_t batch, int32_t active, int32_t T, int32_t H, int32_t G,
                   int32_t Dm, int32_t N, int dt_softplus, int32_t *err_flags)
{
    if (!x || !A || !B || !C || !dt || !pool || !out)
        return 1;
    if (!valid_dtype(x_dt) || !valid_dtype(bc_dt) || !valid_dtype(state_dt))
        return 3;
    if (check_common(batch, active, H, G, Dm, N, slot_stride) || T < 0)
        return 2;
    int given = (st_DA != 0) + (st_U != 0) + (st_B != 0) + (st_DT != 0);
    if (given != 0 && given != 4)
        return 1;
    int stash = given == 4;
    int32_t err = 0;
    const int heads_per_group = H / G;
    const int64_t units = (int64_t)active * H;
    /* every (row, head) unit owns its state block, output rows and stash entries (the
     * stash's B of a group is written by the group's first head) */
#pragma omp parallel for schedule(dynamic, 1) reduction(|:err)
    for (int64_t u = 0; u < units; ++u) {
        const int32_t b = (int32_t)(u / H);
        const int h = (int)(u % H);
        int64_t s = resolve_slot(state_indices, b, P, &err);
        if (s == -1) {                       /* padding row: every position outputs 0 */
            for (int32_t t = 0; t < T; ++t)
                for (int d = 0; d < Dm; ++d)
                    out[(((int64_t)b * T + t) * H + h) * Dm + d] = 0.0;
            continue;
        }
        if (s < 0)
            continue;
        int32_t L = context_lengths ? context_lengths[b] : T;
        if (L > T) {
            err |= 4;
            L = T;
        }
        if (L < 0) {
            err |= 8;
            L = 0;
        }
        if (L == 0)
            continue;
        int g = h / heads_per_group;
        double *S = malloc(sizeof(double) * (size_t)Dm * N);
        for (int64_t i = 0; i < (int64_t)Dm * N; ++i)
            S[i] = load(pool, state_dt, s * slot_stride + (int64_t)h * Dm * N + i);
        for (int32_t t = 0; t < L; ++t) {
            int64_t bt = (int64_t)b * T + t;
            double dte = effective_dt(dt[bt * H + h], dt_bias, h, dt_softplus);
            double decay = exp((double)A[h] * dte);
            if (stash) {
                st_DA[bt * H + h] = (float)decay;
                st_DT[bt * H + h] = (float)dte;
                if (h % heads_per_group == 0)
                    for (int n = 0; n < N; ++n)
                        st_B[(bt * G + g) * N + n] = (float)load(B, bc_dt, (bt * G + g) * N + n);
            }
            for (int d = 0; d < Dm; ++d) {
                int64_t xi = (bt * H + h) * Dm + d;
                double xv = load(x, x_dt, xi);
                if (stash)
                    st_U[xi] = (float)xv;
                double y = 0.0;
                for (int n = 0; n < N; ++n) {
                    int64_t bi = (bt * G + g) * N + n;
                    double *sp = &S[(int64_t)d * N + n];
                    *sp = *sp * decay + load(B, bc_dt, bi) * dte * xv;
                    y += *sp * load(C, bc_dt, bi);
                }
                if (D)
                    y += (double)D[h] * xv;
                if (z)
                    y *= silu(load(z, x_dt, xi));
                out[xi] = y;
            }
        }
        if (!stash)
            for (int64_t i = 0; i < (int64_t)Dm * N; ++i)
                store(pool, state_dt, s * slot_stride + (int64_t)h * Dm * N + i, S[i]);
        free(S);
    }
    if (err_flags)
        *err_flags |= err;
    return 0;
}

/* ---------------- replay of accepted tokens ----------------
 * Selective State Update page, struct MambaReplayLayerInfo and
 * invokeMambaReplayReconstructBatched: re-run the recurrence over the first
 * acceptedLengths[b] stashed tokens, in place on the committed state; a count of 0
 * leaves the row untouched; rows b >= activeBatchSize are not visited.
 *
 * With acceptedNodeIds ([activeBatch, maxAcceptLen], the tree-accept form of the same
 * call) the t-th replayed token is stash entry acceptedNodeIds[b][t] instead of t, and
 * the accepted count is bounded by maxAcceptLen. A node id outside [0, T) among the
 * first acceptedLengths[b] leaves the whole row untouched and sets flag 64. */
int oracle_replay(void *pool, int state_dt, int64_t slot_stride, int32_t P,
                  const float *st_DA, const float *st_U, const float *st_B,
                  const float *st_DT, const int32_t *accepted_lengths,
                  const int32_t *state_indices, int32_t batch, int32_t active, int32_t T,
                  int32_t H, int32_t G, int32_t Dm, int32_t N,
                  const int32_t *node_ids, int32_t max_accept_len, int32_t *err_flags)
{
    if (!pool || !st_DA || !st_U || !st_B || !st_DT || !accepted_lengths)
        return 1;
    if (!valid_dtype(state_dt))
        return 3;
    if (check_common(batch, active, H, G, Dm, N, slot_stride) || T < 0)
        return 2;
    if (node_ids && max_accept_len < 0)
        return 2;
    const int32_t bound = node_ids ? max_accept_len : T;
    int32_t err = 0;
    const int heads_per_group = H / G;
    const int64_t units = (int64_t)active * H;
    /* every (row, head) unit owns its state block */
#pragma omp parallel for schedule(dynamic, 1) reduction(|:err)
    for (int64_t u = 0; u < units; ++u) {
        const int32_t b = (int32_t)(u / H);
        const int h = (int)(u % H);
        int64_t s = resolve_slot(state_indices, b, P, &err);
        if (s < 0)
            continue;                        /* padding row or bad index: no state */
        int32_t k = accepted_lengths[b];
        if (k > bound) {
            err |= 2;
            k = bound;
        }
        if (k < 0) {
            err |= 8;
            k = 0;
        }
        int ids_ok = 1;
        for (int32_t t = 0; node_ids && t < k; ++t) {
            int32_t id = node_ids[(int64_t)b * max_accept_len + t];
            if (id < 0 || id >= T)
                ids_ok = 0;
        }
        if (!ids_ok) {
            err |= 64;
            continue;
        }
        if (k == 0)
            continue;
        int g = h / heads_per_group;
        double *S = malloc(sizeof(double) * (size_t)Dm * N);
        for (int64_t i = 0; i < (int64_t)Dm * N; ++i)
            S[i] = load(pool, state_dt, s * slot_stride + (int64_t)h * Dm * N + i);
        for (int32_t t = 0; t < k; ++t) {
            int32_t e = node_ids ? node_ids[(int64_t)b * max_accept_len + t] : t;
            int64_t bt = (int64_t)b * T + e;
            double decay = st_DA[bt * H + h];
            double dte = st_DT[bt * H + h];
            for (int d = 0; d < Dm; ++d) {
                double uv = st_U[(bt * H + h) * Dm + d];
                for (int n = 0; n < N; ++n) {
                    double *sp = &S[(int64_t)d * N + n];
                    *sp = *sp * decay + (double)st_B[(bt * G + g) * N + n] * dte * uv;
                }
            }
        }
        for (int64_t i = 0; i < (int64_t)Dm * N; ++i)
            store(pool, state_dt, s * slot_stride + (int64_t)h * Dm * N + i, S[i]);
        free(S);
    }
    if (err_flags)
        *err_flags |= err;
    return 0;
}

/* ---------------- tree verify (DDTree) ----------------
 * Selective State Update page, mamba_ssm::invokeSelectiveStateUpdateDDTree: the committed
 * state stays read-only; for every verify node i of row b the ancestors are found by
 * following treeParentIds from i to the root, the recurrence is run from the committed
 * state over that path in root-to-node order, node i's output is taken from the state
 * reached at i, and node i's own (dA, x, B, dt) tuple is stored in the replay stash at
 * position i. Paths stay within the verify budget of 128 nodes.
 *
 * x [batch,T,H,Dm], B/C [batch,T,G,N], dt [batch,T,H], out [batch,T,H,Dm] (no z gate in
 * this call), treeParentIds/treeDepths [batch,T]. Readings: parent -1 attaches a node to
 * the committed state; treeDepths[b][i] counts the tree ancestors of node i, so the walk
 * from i takes exactly that many parent steps and must then reach parent -1. A node whose
 * walk leaves [0, T), ends early or does not end there is malformed: its outputs are 0
 * and flag 64 is set (its stash entry is written like any other). Padding rows output 0
 * at every node and write no stash; an index >= P skips the row (flag 1). */
int oracle_ddtree(const void *x, int x_dt, const float *A, const void *B, const void *C,
                  int bc_dt, const float *dt, const float *dt_bias, const float *D,
                  const void *pool, int state_dt, int64_t slot_stride, int32_t P,
                  double *out, const int32_t *parent_ids, const int32_t *depths,
                  const int32_t *state_indices, float *st_DA, float *st_U, float *st_B,
                  float *st_DT, int32_t batch, int32_t active, int32_t T, int32_t H,
                  int32_t G, int32_t Dm, int32_t N, int dt_softplus, int32_t *err_flags)
{
    if (!x || !A || !B || !C || !dt || !pool || !out || !parent_ids || !depths)
        return 1;
    if (!st_DA || !st_U || !st_B || !st_DT)
        return 1;
    if (!valid_dtype(x_dt) || !valid_dtype(bc_dt) || !valid_dtype(state_dt))
        return 3;
    if (check_common(batch, active, H, G, Dm, N, slot_stride) || T < 0 || T > 128)
        return 2;
    int32_t err = 0;
    const int heads_per_group = H / G;
    const int64_t units = (int64_t)active * H;
    /* every (row, head) unit owns its output rows and stash entries (the stash's B of a
     * group is written by the group's first head); the pool is only read */
#pragma omp parallel for schedule(dynamic, 1) reduction(|:err)
    for (int64_t u = 0; u < units; ++u) {
        const int32_t b = (int32_t)(u / H);
        const int h = (int)(u % H);
        int64_t s = resolve_slot(state_indices, b, P, &err);
        if (s == -1) {                       /* padding row: every node outputs 0 */
            for (int32_t i = 0; i < T; ++i)
                for (int d = 0; d < Dm; ++d)
                    out[(((int64_t)b * T + i) * H + h) * Dm + d] = 0.0;
            continue;
        }
        if (s < 0)
            continue;
        int g = h / heads_per_group;
        /* the stash: every node's own replay inputs */
        for (int32_t i = 0; i < T; ++i) {
            int64_t bi = (int64_t)b * T + i;
            double dte = effective_dt(dt[bi * H + h], dt_bias, h, dt_softplus);
            st_DA[bi * H + h] = (float)exp((double)A[h] * dte);
            st_DT[bi * H + h] = (float)dte;
            for (int d = 0; d < Dm; ++d)
                st_U[(bi * H + h) * Dm + d] = (float)load(x, x_dt, (bi * H + h) * Dm + d);
            if (h % heads_per_group == 0)
                for (int n = 0; n < N; ++n)
                    st_B[(bi * G + g) * N + n] = (float)load(B, bc_dt, (bi * G + g) * N + n);
        }
        double *S = malloc(sizeof(double) * (size_t)Dm * N);
        int32_t path[128];
        for (int32_t i = 0; i < T; ++i) {
            int64_t bi = (int64_t)b * T + i;
            /* walk from node i to the root: path[0] = i, path[k] = k-th ancestor */
            int32_t depth = depths[bi];
            int ok = depth >= 0 && depth < 128;
            int32_t node = i;
            for (int32_t k = 0; ok && k <= depth; ++k) {
                path[k] = node;
                int32_t par = parent_ids[(int64_t)b * T + node];
                if (k < depth) {
                    if (par < 0 || par >= T)
                        ok = 0;
                    node = par;
                } else if (par != -1) {
                    ok = 0;
                }
            }
            if (!ok) {
                err |= 64;
                for (int d = 0; d < Dm; ++d)
                    out[(bi * H + h) * Dm + d] = 0.0;
                continue;
            }
            for (int64_t e = 0; e < (int64_t)Dm * N; ++e)
                S[e] = load(pool, state_dt, s * slot_stride + (int64_t)h * Dm * N + e);
            for (int32_t k = depth; k >= 0; --k) {   /* root-to-node order */
                int64_t bj = (int64_t)b * T + path[k];
                double dte = effective_dt(dt[bj * H + h], dt_bias, h, dt_softplus);
                double decay = exp((double)A[h] * dte);
                for (int d = 0; d < Dm; ++d) {
                    double xv = load(x, x_dt, (bj * H + h) * Dm + d);
                    for (int n = 0; n < N; ++n) {
                        double *sp = &S[(int64_t)d * N + n];
                        *sp = *sp * decay + load(B, bc_dt, (bj * G + g) * N + n) * dte * xv;
                    }
                }
            }
            for (int d = 0; d < Dm; ++d) {
                double y = 0.0;
                for (int n = 0; n < N; ++n)
                    y += S[(int64_t)d * N + n] * load(C, bc_dt, (bi * G + g) * N + n);
                if (D)
                    y += (double)D[h] * load(x, x_dt, (bi * H + h) * Dm + d);
                out[(bi * H + h) * Dm + d] = y;
            }
        }
        free(S);
    }
    if (err_flags)
        *err_flags |= err;
    return 0;
}

/* ---------------- causal conv1d update fused with the decode ----------------
 * The conv state of a slot holds the last width-1 raw inputs of every channel of the
 * concatenated xBC input (conv_dim = H*Dm + 2*G*N channels, order x, B, C): Selective
 * State Update page, struct MambaStateLayerInfo (convState beside recurrentState), and
 * the causal conv1d update of the FlashInfer page flashinfer.gdn_fused_decode_step
 * (conv_weight [dim, width], conv_bias [dim], conv_state [P, dim, width-1] of raw inputs,
 * updated in place, both pools indexed by the same state index, padding rows skipped).
 * Per channel c of an active row with slot s:
 *     window  = (state[s,c,0], ..., state[s,c,width-2], xbc[b,c])     oldest first
 *     v[c]    = sum_k weight[c,k] * window[k] + bias[c],  then v *= sigmoid(v) if conv_silu
 *     state[s,c,:] = window[1..width-1]
 * and the decode of oracle_decode runs with x = v[0 : H*Dm], B = v[H*Dm : H*Dm+G*N],
 * C = v[H*Dm+G*N : conv_dim] (conv outputs kept in double, never rounded). Element (s,c,k)
 * of the conv pool sits at s*conv_slot_stride + c*stride_c + k*stride_k. */
int oracle_conv_decode(const void *xbc, int x_dt, const void *conv_w, const void *conv_b,
                       void *conv_state, int64_t conv_slot_stride, int64_t stride_c,
                       int64_t stride_k, int32_t width, int conv_silu, const float *A,
                       const float *dt, const float *dt_bias, const float *D, const void *z,
                       void *pool, int state_dt, int64_t slot_stride, int32_t P, double *out,
                       const int32_t *state_indices, int32_t batch, int32_t active, int32_t H,
                       int32_t G, int32_t Dm, int32_t N, int dt_softplus, int32_t *err_flags)
{
    if (!xbc || !conv_w || !A || !dt || !pool || !out || (width > 1 && !conv_state))
        return 1;
    if (!valid_dtype(x_dt) || !valid_dtype(state_dt))
        return 3;
    if (check_common(batch, active, H, G, Dm, N, slot_stride) || width < 1)
        return 2;
    const int64_t cd = (int64_t)H * Dm + 2 * (int64_t)G * N;
    int32_t err = 0;
    const int hpg = H / G;
    /* every row owns its slot of both pools and its output rows (the B and C channels of
     * a row are shared by its heads, so the unit of parallel work is the row) */
#pragma omp parallel for schedule(dynamic, 1) reduction(|:err)
    for (int32_t b = 0; b < active; ++b) {
        int64_t s = resolve_slot(state_indices, b, P, &err);
        if (s == -1) {
            for (int64_t i = 0; i < (int64_t)H * Dm; ++i)
                out[(int64_t)b * H * Dm + i] = 0.0;
            continue;
        }
        if (s < 0)
            continue;
        double *v = malloc(sizeof(double) * (size_t)cd);
        double *win = malloc(sizeof(double) * (size_t)width);
        for (int64_t c = 0; c < cd; ++c) {
            for (int k = 0; k + 1 < width; ++k)
                win[k] = load(conv_state, x_dt, s * conv_slot_stride + c * stride_c + k * stride_k);
            win[width - 1] = load(xbc, x_dt, (int64_t)b * cd + c);
            double acc = conv_b ? load(conv_b, x_dt, c) : 0.0;
            for (int k = 0; k < width; ++k)
                acc += load(conv_w, x_dt, c * width + k) * win[k];
            v[c] = conv_silu ? acc / (1.0 + exp(-acc)) : acc;
            for (int k = 0; k + 1 < width; ++k)
                store(conv_state, x_dt, s * conv_slot_stride + c * stride_c + k * stride_k,
                      win[k + 1]);
        }
        for (int h = 0; h < H; ++h) {
            int g = h / hpg;
            double dte = effective_dt(dt[(int64_t)b * H + h], dt_bias, h, dt_softplus);
            double decay = exp((double)A[h] * dte);
            const double *Bv = v + (int64_t)H * Dm + (int64_t)g * N;
            const double *Cv = v + (int64_t)H * Dm + (int64_t)G * N + (int64_t)g * N;
            for (int d = 0; d < Dm; ++d) {
                double xv = v[(int64_t)h * Dm + d];
                double y = 0.0;
                for (int n = 0; n < N; ++n) {
                    int64_t si = s * slot_stride + ((int64_t)h * Dm + d) * N + n;
                    double sn = load(pool, state_dt, si) * decay + Bv[n] * dte * xv;
                    store(pool, state_dt, si, sn);
                    y += sn * Cv[n];
                }
                if (D)
                    y += (double)D[h] * xv;
                int64_t oi = ((int64_t)b * H + h) * Dm + d;
                if (z)
                    y *= silu(load(z, x_dt, oi));
                out[oi] = y;
            }
        }
        free(v);
        free(win);
    }
    if (err_flags)
        *err_flags |= err;
    return 0;
}

/* ---------------- gated delta-rule decode (GDN core) ----------------
 * FlashInfer page flashinfer.gdn_fused_decode_step, its recurrent core: a paged fp32
 * state pool [P, HV, V, K] (V-major, K-last, padded slot stride allowed), state_indices
 * shared with the padding contract above (negative: no state access, output 0; >= P: row
 * skipped, flag 1). Per active row b and value head hv (key head hk = hv / (HV / HK)):
 *     q, k      the key head's query and key (K values); with use_l2norm each is divided
 *               by sqrt(sum of squares + 1e-6); q is then multiplied by scale
 *     g         = -exp(A_log[hv]) * softplus(a[b,hv] + dt_bias[hv]);  alpha = exp(g)
 *     beta      = sigmoid(bgate[b,hv])
 *     S         = alpha * S                         (decay of the whole head state)
 *     for every row i < V:  u = sum_j S[i][j] k[j];  d = beta * (v[i] - u);
 *                           S[i][j] += d * k[j];     out[i] = sum_j S[i][j] q[j]
 * The state is stored back rounded to fp32; out is returned in double. */
int oracle_gdn_decode(const void *q, const void *k, const void *v, int x_dt,
                      const void *a_in, const void *b_in, const float *A_log,
                      const float *dt_bias, double scale, int use_l2norm, float *pool,
                      int64_t slot_stride, int32_t P, double *out,
                      const int32_t *state_indices, int32_t batch, int32_t active, int32_t HK,
                      int32_t HV, int32_t K, int32_t V, int32_t *err_flags)
{
    if (!q || !k || !v || !a_in || !b_in || !A_log || !pool || !out)
        return 1;
    if (!valid_dtype(x_dt))
        return 3;
    if (batch < 0 || active < 0 || active > batch || HK <= 0 || HV <= 0 || HV % HK != 0 ||
        K <= 0 || V <= 0 || slot_stride < (int64_t)HV * V * K)
        return 2;
    int32_t err = 0;
    const int vpk = HV / HK;
    const int64_t units = (int64_t)active * HV;
    /* every (row, value head) unit owns its state block and output row */
#pragma omp parallel for schedule(dynamic, 1) reduction(|:err)
    for (int64_t u = 0; u < units; ++u) {
        const int32_t b = (int32_t)(u / HV);
        const int hv = (int)(u % HV);
        int64_t s = resolve_slot(state_indices, b, P, &err);
        if (s == -1) {
            for (int i = 0; i < V; ++i)
                out[((int64_t)b * HV + hv) * V + i] = 0.0;
            continue;
        }
        if (s < 0)
            continue;
        double *S = malloc(sizeof(double) * (size_t)V * K);
        double *qn = malloc(sizeof(double) * (size_t)K);
        double *kn = malloc(sizeof(double) * (size_t)K);
        int hk = hv / vpk;
        double nq = 0.0, nk = 0.0;
        for (int j = 0; j < K; ++j) {
            qn[j] = load(q, x_dt, ((int64_t)b * HK + hk) * K + j);
            kn[j] = load(k, x_dt, ((int64_t)b * HK + hk) * K + j);
            nq += qn[j] * qn[j];
            nk += kn[j] * kn[j];
        }
        double fq = use_l2norm ? 1.0 / sqrt(nq + 1e-6) : 1.0;
        double fk = use_l2norm ? 1.0 / sqrt(nk + 1e-6) : 1.0;
        for (int j = 0; j < K; ++j) {
            qn[j] *= fq * scale;
            kn[j] *= fk;
        }
        double av = load(a_in, x_dt, (int64_t)b * HV + hv) + (dt_bias ? dt_bias[hv] : 0.0);
        double g = -exp((double)A_log[hv]) * softplus(av);
        double alpha = exp(g);
        double beta = 1.0 / (1.0 + exp(-load(b_in, x_dt, (int64_t)b * HV + hv)));
        int64_t base = s * slot_stride + (int64_t)hv * V * K;
        for (int64_t e = 0; e < (int64_t)V * K; ++e)
            S[e] = alpha * (double)pool[base + e];
        for (int i = 0; i < V; ++i) {
            double *row = S + (int64_t)i * K;
            double uk = 0.0;
            for (int j = 0; j < K; ++j)
                uk += row[j] * kn[j];
            double d = beta * (load(v, x_dt, ((int64_t)b * HV + hv) * V + i) - uk);
            double o = 0.0;
            for (int j = 0; j < K; ++j) {
                row[j] += d * kn[j];
                o += row[j] * qn[j];
            }
            out[((int64_t)b * HV + hv) * V + i] = o;
        }
        for (int64_t e = 0; e < (int64_t)V * K; ++e)
            pool[base + e] = (float)S[e];
        free(S);
        free(qn);
        free(kn);
    }
    if (err_flags)
        *err_flags |= err;
    return 0;
}

/* ---------------- thread count ----------------
 * The loops above run their independent units (a row and head, or a row) on the
 * OpenMP threads; each unit's arithmetic is sequential and in the same order for any
 * thread count, so results do not depend on it. n <= 0 selects every host core. */
void oracle_set_threads(int n) { omp_set_num_threads(n > 0 ? n : omp_get_num_procs()); }

int oracle_max_threads(void) { return omp_get_max_threads(); }

int oracle_host_cores(void) { return omp_get_num_procs(); }

/* ---------------- slot maintenance ----------------
 * Selective State Update page, invokeMambaStateClear (one slot, or all when slot is -1)
 * and Recurrent State Manager page, clearSlot / copySlotFrom. */
int oracle_clear_slot(void *pool, int64_t slot_bytes, int32_t P, int32_t slot)
{
    if (!pool || slot_bytes < 0 || P < 0 || slot < -1 || slot >= P)
        return 2;
    if (slot == -1)
        memset(pool, 0, (size_t)slot_bytes * (size_t)P);
    else
        memset((char *)pool + (int64_t)slot * slot_bytes, 0, (size_t)slot_bytes);
    return 0;
}

int oracle_copy_slot(void *dst_pool, int32_t dst_P, int32_t dst_slot,
                     const void *src_pool, int32_t src_P, int32_t src_slot,
                     int64_t slot_bytes)
{
    if (!dst_pool || !src_pool || slot_bytes < 0)
        return 2;
    if (dst_slot < 0 || dst_slot >= dst_P || src_slot < 0 || src_slot >= src_P)
        return 2;
    memmove((char *)dst_pool + (int64_t)dst_slot * slot_bytes,
            (const char *)src_pool + (int64_t)src_slot * slot_bytes, (size_t)slot_bytes);
    return 0;
}

/* ---------------- multi-layer launches and gather/scatter ----------------
 * Selective State Update page: invokeMambaReplayReconstructBatched over an array of
 * MambaReplayLayerInfo (every layer replays its own stash into its own pool, sharing
 * acceptedLengths and stateIndices), invokeMambaStateClear over MambaStateLayerInfo
 * (recurrent and convolution states of every layer), and invokeMambaStateGather /
 * Scatter (copy active rows between the resident pool and a contiguous batch). */
int oracle_replay_layers(void *const *pools, const float *const *st_DA,
                         const float *const *st_U, const float *const *st_B,
                         const float *const *st_DT, int32_t num_layers, int state_dt,
                         int64_t slot_stride, int32_t P, const int32_t *accepted_lengths,
                         const int32_t *state_indices, int32_t batch, int32_t active,
                         int32_t T, int32_t H, int32_t G, int32_t Dm, int32_t N,
                         const int32_t *node_ids, int32_t max_accept_len, int32_t *err_flags)
{
    for (int32_t l = 0; l < num_layers; ++l) {
        int rc = oracle_replay(pools[l], state_dt, slot_stride, P, st_DA[l], st_U[l], st_B[l],
                               st_DT[l], accepted_lengths, state_indices, batch, active, T, H,
                               G, Dm, N, node_ids, max_accept_len, err_flags);
        if (rc)
            return rc;
    }
    return 0;
}

int oracle_clear_slot_layers(void *const *recurrent, void *const *conv, int32_t num_layers,
                             int32_t P, int32_t slot, int64_t recurrent_slot_bytes,
                             int64_t conv_slot_bytes)
{
    for (int32_t l = 0; l < num_layers; ++l) {
        if (recurrent[l] && recurrent_slot_bytes) {
            int rc = oracle_clear_slot(recurrent[l], recurrent_slot_bytes, P, slot);
            if (rc)
                return rc;
        }
        if (conv && conv[l] && conv_slot_bytes) {
            int rc = oracle_clear_slot(conv[l], conv_slot_bytes, P, slot);
            if (rc)
                return rc;
        }
    }
    return 0;
}

/* scatter == 0: dense[b] = pool[slot(b)], zeros for a padding row;
 * scatter != 0: pool[slot(b)] = dense[b], nothing for a padding row;
 * an index >= P skips the row and sets bit 1. */
int oracle_gather_scatter(void *pool, int64_t slot_bytes, int32_t P, void *dense,
                          const int32_t *state_indices, int32_t batch, int32_t active,
                          int scatter, int32_t *err_flags)
{
    if (!pool || !dense || slot_bytes < 0 || active < 0 || active > batch)
        return 2;
    int32_t err = 0;
    for (int32_t b = 0; b < active; ++b) {
        int64_t s = state_indices ? state_indices[b] : b;
        char *drow = (char *)dense + (int64_t)b * slot_bytes;
        if (s >= P) {
            err |= 1;
            continue;
        }
        if (s < 0) {
            if (!scatter)
                memset(drow, 0, (size_t)slot_bytes);
            continue;
        }
        char *prow = (char *)pool + s * slot_bytes;
        if (scatter)
            memcpy(prow, drow, (size_t)slot_bytes);
        else
            memcpy(drow, prow, (size_t)slot_bytes);
    }
    if (err_flags)
        *err_flags |= err;
    return 0;
}
