// ssu_ddtree.cu -- tree verify: the output of every node of a draft tree, each from the
// committed state along its own ancestor path, in one launch.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API),
// mamba_ssm::invokeSelectiveStateUpdateDDTree: the committed state stays read-only; for
// every verify node the recurrence runs from the committed state over the node's
// ancestor path in root-to-node order, the node's output is taken there, and the node's
// own (dA, x, B, dt) tuple goes to the replay stash for the accepted-path commit. Trees
// hold at most 128 nodes.
//
// Walking every path separately would cost one full state update per path node. The
// kernel unrolls the recurrence along the path j_0 .. j_k = i instead:
//     s_i = W_i * s0 + sum_m w_im * dt_jm * x_jm * B_jm,
//     w_im = product of dA_jl over l > m,   W_i = product of dA over the whole path,
// so that with a_i = s0 . C_i (one dot product over dstate per dim row)
//     out_i = W_i * a_i + sum_m w_im * dt_jm * (C_i . B_jm) * x_jm + D * x_i.
// The only dense work is a_i, dim x dstate multiply-adds per node and head (one decode
// step without its state write); the path sums cost (path length) x (dim + dstate). No
// node's state is ever formed and nothing is written to the pool.
//
// Two forms compute the same outputs and stash: with bf16 B and C and dstate 64 or 128 the
// dense products run on the tcgen05 tensor cores (the tensor-core form further down);
// for every other type the CUDA-core form described here runs.
//
// Work items are (row, head, 64-row dim tile), row-major. A persistent CTA of 8 warps
// takes a contiguous range of items, so consecutive items share their row's tree and its
// C . B products, built once per (row, group) in shared memory:
//   * parents of the row, each node's path checked (exactly depth parent steps, then
//     parent -1; otherwise the node is malformed: outputs 0, SSU_FLAG_TREE);
//   * C of every node widened to fp32 (rows padded against bank conflicts);
//   * for every node i and every node j_m on its path: j_m and cb = C_i . B_jm.
// The committed-state rows of the next item and its x tile are fetched by cp.async while
// the current item computes: coalesced 16-byte copies into shared memory (the state rows
// with an XOR swizzle of their 16-byte chunks, so that the row-per-lane reads below are
// free of bank conflicts; the x tile double-buffered when it fits), and the next item's
// dt is loaded into registers early. Per item: the path coefficients w_im * dt_jm * cb
// and W_i are formed once per node, then all path sums P[i][d] in one parallel pass (a
// thread per node and half tile, 32 sums in registers); the dense products run with the
// lane mapping described at TGeo, a transposing shuffle reduction leaves each lane with
// whole rows, and out = W_i a_i + P[i][d] + D x is stored without further barriers.
#include <type_traits>

#include "ssu_async.cuh"
#include "ssu_common.cuh"
#include "ssu_tc.cuh"
#include "ssu_tmap.cuh"

namespace ssu {
namespace {

constexpr int kThreads = 256;      // 8 warps, one CTA per SM
constexpr int kTile = 64;          // dim rows per work item
constexpr int kMaxNodes = 128;     // the verify budget
constexpr int kSmemMax = 227 * 1024;
constexpr int kBatch = 8;          // loads in flight per thread in the plain-load loops
constexpr int kXS = kTile + 8;     // x tile row stride (elements): rows start in different banks

// Lane mapping of the dense products: the warp's lanes form QG column groups of LG lanes
// (quarter warps at dstate >= 128); a lane holds R state rows over the K columns of its
// group, interleaved in 16-byte groups (group q owns float4 column groups q, q + QG, ..).
// All lanes of a group read the same C address and the groups read adjacent 16-byte
// chunks, which costs the shared-memory pipe what a warp-wide broadcast costs (2.56 SM
// cycles per warp-wide 16-byte load on B200, measured) while delivering QG times the
// data, and every C value loaded serves R rows. RWT warps cover a 64-row tile; the
// NG = 8 / RWT node groups take every NG-th node.
template <int N> struct TGeo {
    static constexpr int QG = N >= 128 ? 4 : (N == 64 ? 2 : 1);   // column groups
    static constexpr int LG = 32 / QG;                  // lanes per column group
    static constexpr int K = N / QG;                    // state columns per lane
    static constexpr int R = N == 256 ? 2 : (N >= 64 ? 4 : 2);      // rows per lane
    static constexpr int RW = LG * R;                   // rows per warp
    static constexpr int RWT = kTile / RW;              // warps per 64-row tile
    static constexpr int NG = kThreads / 32 / RWT;      // node groups
    static constexpr int NOWN = QG == 4 ? 1 : (QG == 2 ? R / 2 : R);  // rows a lane finishes
    static constexpr int CP = N + 4;                    // padded fp32 row of C (floats)
    static_assert(RW * RWT == kTile && K % 4 == 0 && K * R <= 128 && NG >= 1,
                  "tree geometry");
};

// Shared-memory layout (byte offsets, 16-byte aligned). E = T (T + 1) / 2 bounds the
// number of (node, path node) pairs; nxb x tiles (2: the next item's is prefetched).
struct TLayout {
    int cf, s0, xs, xbytes, cb, coef, pj, par, cnt, off, da, dtv, wt, total;
    __host__ __device__ static int up16(int v) { return (v + 15) & ~15; }
    __host__ __device__ TLayout(int T, int N, int es_x, int es_s, int nxb)
    {
        const int E = T * (T + 1) / 2;
        cf = 0;
        s0 = cf + up16(T * (N + 4) * 4);
        xs = s0 + up16(kTile * N * es_s);
        xbytes = up16(T * kXS * es_x);
        cb = xs + nxb * xbytes;
        coef = cb + up16(E * 4);
        // the coefficients of an item, then its path sums [T][kTile] in the same bytes
        pj = coef + up16(E * 4 > T * kTile * 4 ? E * 4 : T * kTile * 4);
        par = pj + up16(E);
        cnt = par + up16(T * 4);
        off = cnt + up16(T * 4);
        da = off + up16(T * 4);
        dtv = da + up16(T * 4);
        wt = dtv + up16(T * 4);
        total = wt + up16(T * 4);
    }
};

// Byte offset of 16-byte chunk c of state row r in the staging buffer (cpr chunks per
// row): chunks are XOR-swizzled by the row so that lanes reading the same chunk of
// consecutive rows hit different banks.
__device__ __forceinline__ int s0_off(int r, int c, int cpr)
{
    const int m = (cpr < 8 ? cpr : 8) - 1;
    return (r * cpr + (c ^ (r & m))) * 16;
}

// One work item: row b, head h (group g), dim rows row0 .. row0 + rows, pool slot.
struct Item {
    int b, h, g, dtile, row0, rows, slot;
    __device__ __forceinline__ bool valid(int P) const { return slot >= 0 && slot < P; }
};

__device__ __forceinline__ Item item_at(const TreeArgs &ta, int64_t it, int dtiles)
{
    const DecodeArgs &a = ta.d;
    Item u;
    u.dtile = (int)(it % dtiles);
    u.h = (int)((it / dtiles) % a.H);
    u.b = (int)(it / ((int64_t)dtiles * a.H));
    u.g = u.h / (a.H / a.G);
    u.row0 = u.dtile * kTile;
    u.rows = min(kTile, a.Dm - u.row0);
    u.slot = a.idx ? a.idx[u.b] : u.b;
    return u;
}

// The pool slot of row b (-1 past the active rows).
__device__ __forceinline__ int row_slot(const TreeArgs &ta, int b)
{
    const DecodeArgs &a = ta.d;
    return b < a.active ? (a.idx ? a.idx[b] : b) : -1;
}

// The item after u in row-major order, with the slot of the next row prefetched in nslot:
// at a row change the row takes it, and the slot of the row after is loaded, a whole row
// ahead of its use.
__device__ __forceinline__ Item item_after_pf(const TreeArgs &ta, const Item &u, int dtiles,
                                              int &nslot)
{
    const DecodeArgs &a = ta.d;
    Item v = u;
    if (++v.dtile == dtiles) {
        v.dtile = 0;
        if (++v.h == a.H) {
            v.h = 0;
            ++v.b;
            v.slot = nslot;
            nslot = row_slot(ta, v.b + 1);
        }
        v.g = v.h / (a.H / a.G);
    }
    v.row0 = v.dtile * kTile;
    v.rows = min(kTile, a.Dm - v.row0);
    return v;
}

// C_i . B_j over dstate: C_i from shared memory (fp32), B_j from global memory (16-byte
// rows of the input type).
template <int N>
__device__ __forceinline__ float dot_cb(const float *ci, const void *B, int dtype,
                                        int64_t base)
{
    float s0 = 0.f, s1 = 0.f;
    if (dtype == SSU_F32) {
        const float4 *bp = reinterpret_cast<const float4 *>(static_cast<const float *>(B) + base);
#pragma unroll 4
        for (int q = 0; q < N / 4; ++q) {
            const float4 bv = __ldg(bp + q);
            const float4 cv = *reinterpret_cast<const float4 *>(ci + 4 * q);
            s0 = fmaf(cv.x, bv.x, s0);
            s1 = fmaf(cv.y, bv.y, s1);
            s0 = fmaf(cv.z, bv.z, s0);
            s1 = fmaf(cv.w, bv.w, s1);
        }
    } else {
        const uint4 *bp =
            reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(B) + base);
#pragma unroll 4
        for (int q = 0; q < N / 8; ++q) {
            const uint4 raw = __ldg(bp + q);
            float f[8];
            if (dtype == SSU_BF16)
                Vec16<__nv_bfloat16>::unpack(raw, f);
            else
                Vec16<__half>::unpack(raw, f);
            const float4 c0 = *reinterpret_cast<const float4 *>(ci + 8 * q);
            const float4 c1 = *reinterpret_cast<const float4 *>(ci + 8 * q + 4);
            s0 = fmaf(c0.x, f[0], s0);
            s1 = fmaf(c0.y, f[1], s1);
            s0 = fmaf(c0.z, f[2], s0);
            s1 = fmaf(c0.w, f[3], s1);
            s0 = fmaf(c1.x, f[4], s0);
            s1 = fmaf(c1.y, f[5], s1);
            s0 = fmaf(c1.z, f[6], s0);
            s1 = fmaf(c1.w, f[7], s1);
        }
    }
    return s0 + s1;
}

// Element e of an x tile held in shared memory in its input type.
__device__ __forceinline__ float xs_at(const uint8_t *xs, int x_dtype, int e)
{
    if (x_dtype == SSU_F32)
        return reinterpret_cast<const float *>(xs)[e];
    return bits_f32(reinterpret_cast<const uint16_t *>(xs)[e], x_dtype);
}

// Shared tables of one (row, group): parents, path checks, C, path nodes and C . B.
template <int N>
__device__ void stage_row(const TreeArgs &ta, const TLayout &lay, uint8_t *sm, int b, int g,
                          bool reporter)
{
    using Gm = TGeo<N>;
    const DecodeArgs &a = ta.d;
    const int T = ta.T, G = a.G, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *Cf = reinterpret_cast<float *>(sm + lay.cf);
    float *cb = reinterpret_cast<float *>(sm + lay.cb);
    uint8_t *pj = sm + lay.pj;
    int *par = reinterpret_cast<int *>(sm + lay.par);
    int *cnt = reinterpret_cast<int *>(sm + lay.cnt);
    int *off = reinterpret_cast<int *>(sm + lay.off);

    for (int i = tid; i < T; i += kThreads)
        par[i] = ta.parents[(int64_t)b * T + i];
    const int64_t cbase = (int64_t)b * T * G * N;
    for (int e0 = tid; e0 < T * N; e0 += kThreads * kBatch) {
        float v[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {       // every load first, then the stores
            const int e = e0 + q * kThreads;
            v[q] = e < T * N ? ld_f32(a.C, a.bc_dtype, cbase + ((int64_t)(e / N) * G + g) * N + e % N)
                             : 0.f;
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int e = e0 + q * kThreads;
            if (e < T * N)
                Cf[(e / N) * Gm::CP + e % N] = v[q];
        }
    }
    __syncthreads();
    // every node's walk: exactly depth parent steps inside [0, T), then parent -1
    for (int i = tid; i < T; i += kThreads) {
        const int depth = ta.depths[(int64_t)b * T + i];
        bool ok = depth >= 0 && depth < kMaxNodes;
        int j = i;
        for (int k = 0; ok && k < depth; ++k) {
            j = par[j];
            ok = j >= 0 && j < T;
        }
        ok = ok && par[j] == -1;
        cnt[i] = ok ? depth + 1 : 0;
        if (!ok && reporter && a.err)
            atomicOr(a.err, SSU_FLAG_TREE);
    }
    __syncthreads();
    if (warp == 0) {                     // exclusive prefix sum of the path lengths
        int carry = 0;
        for (int base = 0; base < T; base += 32) {
            const int i = base + lane;
            const int v = i < T ? cnt[i] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += t;
            }
            if (i < T)
                off[i] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncthreads();
    // path nodes and C_i . B_j: two threads per node, alternate path entries
    for (int t = tid; t < 2 * T; t += kThreads) {
        const int i = t >> 1, p = t & 1, c = cnt[i], o = off[i];
        int j = i;
        for (int k = 0; k < c; ++k) {
            if ((k & 1) == p) {
                pj[o + k] = static_cast<uint8_t>(j);
                cb[o + k] = dot_cb<N>(Cf + i * Gm::CP, a.B, a.bc_dtype,
                                      (((int64_t)b * T + j) * G + g) * N);
            }
            j = par[j];
        }
    }
}

// x tile of item u with plain loads (x rows not 16-byte aligned): rows >= u.rows are 0.
template <int NT>
__device__ void stage_x_plain(const TreeArgs &ta, uint8_t *xs, const Item &u)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, Dm = a.Dm, tid = threadIdx.x;
    for (int e0 = tid; e0 < T * kTile; e0 += NT * kBatch) {
        uint32_t v[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int e = e0 + q * NT, i = e / kTile, d = e % kTile;
            v[q] = e < T * kTile && d < u.rows
                       ? ld_bits(a.x, a.x_dtype, (((int64_t)u.b * T + i) * H + u.h) * Dm + u.row0 + d)
                       : 0u;
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int e = e0 + q * NT, xe = (e / kTile) * kXS + e % kTile;
            if (e < T * kTile) {
                if (a.x_dtype == SSU_F32)
                    reinterpret_cast<uint32_t *>(xs)[xe] = v[q];
                else
                    reinterpret_cast<uint16_t *>(xs)[xe] = static_cast<uint16_t>(v[q]);
            }
        }
    }
}

// Per-head scalars of an item, loaded ahead of their use.
struct HeadVals {
    float A, bias, D;
};

__device__ __forceinline__ HeadVals head_vals(const DecodeArgs &a, int h)
{
    return {a.A[h], a.dt_bias ? a.dt_bias[h] : 0.f, a.D ? a.D[h] : 0.f};
}

// dt_eff and dA of every node for the item's head (node threadIdx.x, from its prefetched
// dt) into shared memory, and into the stash once per (row, head).
__device__ __forceinline__ void node_values(const TreeArgs &ta, float *sdA, float *sdt,
                                            const Item &u, float dt_mine, const HeadVals &hv)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, tid = threadIdx.x;
    if (tid < T) {
        const int64_t bi = (int64_t)u.b * T + tid;
        const float v = dt_mine + hv.bias;
        const float dte = a.softplus ? softplus_f(v) : v;
        const float dA = expf(hv.A * dte);
        sdA[tid] = dA;
        sdt[tid] = dte;
        if (u.dtile == 0) {
            ta.st_dA[bi * a.H + u.h] = dA;
            ta.st_dt[bi * a.H + u.h] = dte;
        }
    }
}

// B of the (row, group) in equal shares by the group's heads (the items of one row are
// spread over the CTAs, so no CTA carries the whole copy).
template <int NT>
__device__ void stash_b(const TreeArgs &ta, const Item &u)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, G = a.G, N = a.N, tid = threadIdx.x;
    if (u.dtile == 0 && tid < NT) {
        // flat element e of the row's [T][N] block: node e / N, column e % N (32-bit
        // arithmetic: T N <= 2^15)
        const int hpg = H / G, hh = u.h % hpg, total = T * N;
        const int e0 = total * hh / hpg, e1 = total * (hh + 1) / hpg;
        const int64_t rbase = ((int64_t)u.b * T * G + u.g) * N;   // node 0 of the row
        const int64_t rstride = (int64_t)G * N;                    // node to node
        for (int eb = e0 + tid; eb < e1; eb += NT * kBatch) {
            float v[kBatch];
            int64_t at[kBatch];
#pragma unroll
            for (int q = 0; q < kBatch; ++q) {
                const int e = eb + q * NT, i = e / N;
                at[q] = rbase + i * rstride + (e - i * N);
                v[q] = e < e1 ? ld_f32(a.B, a.bc_dtype, at[q]) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < kBatch; ++q)
                if (eb + q * NT < e1)
                    ta.st_B[at[q]] = v[q];
        }
    }
}

// Stash of the item: U from the x tile, then its share of B.
template <int NT>
__device__ void stash_ub(const TreeArgs &ta, const Item &u, const uint8_t *xs)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, Dm = a.Dm, tid = threadIdx.x;
    if ((Dm & 3) == 0 && (reinterpret_cast<uintptr_t>(ta.st_U) & 15) == 0) {
        // U: four rows per thread, 16-byte stores
        for (int e = tid; e < T * (kTile / 4); e += NT) {
            const int i = e / (kTile / 4), d = 4 * (e % (kTile / 4));
            if (d < u.rows) {
                float4 f;
                if (a.x_dtype == SSU_F32) {
                    f = *reinterpret_cast<const float4 *>(xs + (i * kXS + d) * 4);
                } else {
                    const uint2 w = *reinterpret_cast<const uint2 *>(xs + (i * kXS + d) * 2);
                    f = make_float4(bits_f32(w.x & 0xffffu, a.x_dtype), bits_f32(w.x >> 16, a.x_dtype),
                                    bits_f32(w.y & 0xffffu, a.x_dtype), bits_f32(w.y >> 16, a.x_dtype));
                }
                *reinterpret_cast<float4 *>(
                    ta.st_U + (((int64_t)u.b * T + i) * H + u.h) * Dm + u.row0 + d) = f;
            }
        }
    } else {
        for (int e = tid; e < T * kTile; e += NT) {
            const int i = e / kTile, d = e % kTile;
            if (d < u.rows)
                ta.st_U[(((int64_t)u.b * T + i) * H + u.h) * Dm + u.row0 + d] =
                    xs_at(xs, a.x_dtype, i * kXS + d);
        }
    }
    stash_b<NT>(ta, u);
}

// Node values and stash of an item (dt of node threadIdx.x prefetched).
__device__ void stage_nodes(const TreeArgs &ta, float *sdA, float *sdt, const Item &u,
                            const uint8_t *xs, float dt_mine)
{
    node_values(ta, sdA, sdt, u, dt_mine, head_vals(ta.d, u.h));
    stash_ub<kThreads>(ta, u, xs);
}

// Path coefficients of the item's head: coef[o_i + m] = w_im * dt_jm * cb[o_i + m], W_i.
__device__ void path_coefs(const TLayout &lay, uint8_t *sm, int T)
{
    const float *cb = reinterpret_cast<const float *>(sm + lay.cb);
    float *coef = reinterpret_cast<float *>(sm + lay.coef);
    const uint8_t *pj = sm + lay.pj;
    const int *cnt = reinterpret_cast<const int *>(sm + lay.cnt);
    const int *off = reinterpret_cast<const int *>(sm + lay.off);
    const float *sdA = reinterpret_cast<const float *>(sm + lay.da);
    const float *sdt = reinterpret_cast<const float *>(sm + lay.dtv);
    float *wt = reinterpret_cast<float *>(sm + lay.wt);
    for (int i = threadIdx.x; i < T; i += kThreads) {
        const int c = cnt[i], o = off[i];
        float w = 1.f;
        for (int k = 0; k < c; ++k) {
            const int j = pj[o + k];
            coef[o + k] = w * sdt[j] * cb[o + k];
            w *= sdA[j];
        }
        wt[i] = w;
    }
}

// Four consecutive committed-state elements of row r (columns col .. col + 3) from the
// swizzled staging buffer.
template <typename S, int N>
__device__ __forceinline__ float4 s0_quad(const uint8_t *buf, int r, int col)
{
    constexpr int cpr = N * (int)sizeof(S) / 16;
    if constexpr (sizeof(S) == 4) {
        return *reinterpret_cast<const float4 *>(buf + s0_off(r, col / 4, cpr));
    } else {
        const int c = col / 8, half = (col / 4) & 1;
        return Quad<S>::load(reinterpret_cast<const S *>(buf + s0_off(r, c, cpr) + half * 8));
    }
}

// Issue the cp.async copies of item u's committed-state rows into the staging buffer.
template <typename S, int N>
__device__ __forceinline__ void prefetch_s0(const TreeArgs &ta, const TLayout &lay, uint8_t *sm,
                                            const Item &u)
{
    const DecodeArgs &a = ta.d;
    constexpr int cpr = N * (int)sizeof(S) / 16;
    const char *src = static_cast<const char *>(a.state) +
                      ((int64_t)u.slot * a.slot_stride + ((int64_t)u.h * a.Dm + u.row0) * N) *
                          (int64_t)sizeof(S);
    for (int k = threadIdx.x; k < u.rows * cpr; k += kThreads)
        cp_async16(sm + lay.s0 + s0_off(k / cpr, k % cpr, cpr), src + (int64_t)k * 16);
}

// Issue the cp.async copies of item u's x tile (rows 16-byte aligned) into buffer xbuf.
// xs_off, xbytes: the buffers' offset and size.
__device__ __forceinline__ void prefetch_x(const TreeArgs &ta, int xs_off, int xbytes, uint8_t *sm,
                                           const Item &u, int xbuf)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, es_x = a.x_dtype == SSU_F32 ? 4 : 2;
    const int cpn = u.rows * es_x / 16;              // 16-byte chunks per node row
    uint8_t *dst = sm + xs_off + xbuf * xbytes;
    const char *xg = static_cast<const char *>(a.x);
    for (int k = threadIdx.x; k < T * cpn; k += kThreads) {
        const int i = k / cpn, c = k % cpn;
        cp_async16(dst + i * kXS * es_x + c * 16,
                   xg + ((((int64_t)u.b * T + i) * a.H + u.h) * a.Dm + u.row0) * es_x + c * 16);
    }
}

// dt of node threadIdx.x for item u (consumed when u is processed).
__device__ __forceinline__ float dt_of(const TreeArgs &ta, const Item &u)
{
    const int T = ta.T;
    return threadIdx.x < T ? ta.d.dt[((int64_t)u.b * T + threadIdx.x) * ta.d.H + u.h] : 0.f;
}

// Path sums of the item: P[i][d] = sum over node i's path entries m of coef[o_i + m] *
// x[j_m][d], for every node and dim row, written over the coefficients (which they no
// longer need). Thread t takes node t / 2 and 32 consecutive rows (half t % 2), keeps the
// 32 sums in registers and reads each path node's x row 16 bytes at a time.
__device__ void path_sums(const TLayout &lay, uint8_t *sm, const uint8_t *xs, int x_dtype,
                          int T)
{
    float *coef = reinterpret_cast<float *>(sm + lay.coef);
    const uint8_t *pj = sm + lay.pj;
    const int *cnt = reinterpret_cast<const int *>(sm + lay.cnt);
    const int *off = reinterpret_cast<const int *>(sm + lay.off);
    const int i = threadIdx.x >> 1, d0 = (threadIdx.x & 1) * 32;
    float acc[32];
#pragma unroll
    for (int e = 0; e < 32; ++e)
        acc[e] = 0.f;
    const int cn = i < T ? cnt[i] : 0, o = i < T ? off[i] : 0;
    for (int k = 0; k < cn; ++k) {
        const float cf = coef[o + k];
        const int j = pj[o + k];
        if (x_dtype == SSU_F32) {
            const float4 *xr = reinterpret_cast<const float4 *>(xs + (j * kXS + d0) * 4);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v = xr[q];
                acc[4 * q] = fmaf(cf, v.x, acc[4 * q]);
                acc[4 * q + 1] = fmaf(cf, v.y, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(cf, v.z, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(cf, v.w, acc[4 * q + 3]);
            }
        } else {
            const uint4 *xr = reinterpret_cast<const uint4 *>(xs + (j * kXS + d0) * 2);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float f[8];
                if (x_dtype == SSU_BF16)
                    Vec16<__nv_bfloat16>::unpack(xr[q], f);
                else
                    Vec16<__half>::unpack(xr[q], f);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    acc[8 * q + e] = fmaf(cf, f[e], acc[8 * q + e]);
            }
        }
    }
    __syncthreads();                     // every coefficient has been read
    if (i < T) {
        float4 *pr = reinterpret_cast<float4 *>(coef + i * kTile + d0);
#pragma unroll
        for (int q = 0; q < 8; ++q)
            pr[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
    }
}

template <typename S, int N>
__global__ void __launch_bounds__(kThreads, 1)
ssu_ddtree_kernel(const __grid_constant__ TreeArgs ta, const int dtiles, const int64_t nitems,
                  const int nxb, const int xasync)
{
    using Gm = TGeo<N>;
    extern __shared__ __align__(16) uint8_t sm[];
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, Dm = a.Dm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ng = warp / Gm::RWT;                   // node group
    const int cg = lane / Gm::LG;                    // column group
    const int rb = (warp % Gm::RWT) * Gm::RW + lane % Gm::LG;   // row of the lane's i = 0
    const int es_x = a.x_dtype == SSU_F32 ? 4 : 2;
    const TLayout lay(T, N, es_x, (int)sizeof(S), nxb);
    const float *Cf = reinterpret_cast<const float *>(sm + lay.cf);
    const float *psum = reinterpret_cast<const float *>(sm + lay.coef);  // path sums [T][64]
    const int *cnt = reinterpret_cast<const int *>(sm + lay.cnt);
    const float *wt = reinterpret_cast<const float *>(sm + lay.wt);

    // Copies for the next item start as early as their buffers allow: the state rows once
    // every lane holds them in registers, the x tile at once when it is double-buffered,
    // else after the item.
    const bool x_mid = xasync && nxb == 2;
    const int64_t first = nitems * blockIdx.x / gridDim.x;
    const int64_t last = nitems * (blockIdx.x + 1) / gridDim.x;
    auto xbuf_of = [&](int64_t it) { return nxb == 2 ? (int)((it - first) & 1) : 0; };
    float dt_next = 0.f;                 // dt of node tid for the next valid item
    if (first < last) {
        const Item u = item_at(ta, first, dtiles);
        if (u.valid(a.P)) {
            prefetch_s0<S, N>(ta, lay, sm, u);
            if (xasync)
                prefetch_x(ta, lay.xs, lay.xbytes, sm, u, xbuf_of(first));
            cp_async_commit();
            dt_next = dt_of(ta, u);
        }
    }
    int cur_b = -1, cur_g = -1;
    for (int64_t it = first; it < last; ++it) {
        const Item u = item_at(ta, it, dtiles);
        const bool has_next = it + 1 < last;
        const Item v = has_next ? item_at(ta, it + 1, dtiles) : u;
        const bool next_valid = has_next && v.valid(a.P);
        if (!u.valid(a.P)) {
            if (u.slot < 0) {            // padding row: zero outputs at every node
                for (int e = tid; e < T * kTile; e += kThreads) {
                    const int i = e / kTile, dd = e % kTile;
                    if (dd < u.rows)
                        st_f32(a.out, a.x_dtype,
                               (((int64_t)u.b * T + i) * H + u.h) * Dm + u.row0 + dd, 0.f);
                }
            } else if (u.h == 0 && u.dtile == 0 && tid == 0 && a.err) {
                atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
            }
            if (next_valid) {            // this item used no buffer: start the next one
                prefetch_s0<S, N>(ta, lay, sm, v);
                if (xasync)
                    prefetch_x(ta, lay.xs, lay.xbytes, sm, v, xbuf_of(it + 1));
                cp_async_commit();
                dt_next = dt_of(ta, v);
            }
            continue;
        }
        uint8_t *xs = sm + lay.xs + xbuf_of(it) * lay.xbytes;
        __syncthreads();                 // the previous item is done with shared memory
        if (u.b != cur_b || u.g != cur_g) {
            stage_row<N>(ta, lay, sm, u.b, u.g, u.h == 0 && u.dtile == 0);
            cur_b = u.b;
            cur_g = u.g;
        }
        if (!xasync)
            stage_x_plain<kThreads>(ta, xs, u);
        cp_async_wait_all();
        __syncthreads();                 // state rows and x tile have landed
        stage_nodes(ta, reinterpret_cast<float *>(sm + lay.da),
                    reinterpret_cast<float *>(sm + lay.dtv), u, xs, dt_next);
        __syncthreads();                 // dt_eff and dA of every node visible
        path_coefs(lay, sm, T);
        __syncthreads();                 // path coefficients and W_i ready
        path_sums(lay, sm, xs, a.x_dtype, T);

        // the lane's R rows of the committed state over its column group
        float2 st[Gm::R][Gm::K / 2];
#pragma unroll
        for (int i = 0; i < Gm::R; ++i) {
            const int r = rb + i * Gm::LG;
#pragma unroll
            for (int j = 0; j < Gm::K / 4; ++j) {
                const float4 f = r < u.rows
                                     ? s0_quad<S, N>(sm + lay.s0, r, 4 * (j * Gm::QG + cg))
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                st[i][2 * j] = make_float2(f.x, f.y);
                st[i][2 * j + 1] = make_float2(f.z, f.w);
            }
        }
        __syncthreads();                 // path sums ready; staging buffer free
        if (next_valid) {
            prefetch_s0<S, N>(ta, lay, sm, v);
            if (x_mid)
                prefetch_x(ta, lay.xs, lay.xbytes, sm, v, xbuf_of(it + 1));
            cp_async_commit();
            dt_next = dt_of(ta, v);
        }
        const float Dh = a.D ? a.D[u.h] : 0.f;

        // y_i = W_i a_i + path sum + D x_i for this warp's nodes, two at a time: partial
        // dot products of the lane's R rows over its columns, then a transposing reduction
        // across the column groups that leaves each lane with whole rows to finish
#pragma unroll 1
        for (int i0 = ng; i0 < T; i0 += 2 * Gm::NG) {
            const int i1 = i0 + Gm::NG;
            const bool two = i1 < T;
            const float *c0 = Cf + i0 * Gm::CP + 4 * cg;
            const float *c1 = Cf + (two ? i1 : i0) * Gm::CP + 4 * cg;
            float2 a0[Gm::R][2], a1[Gm::R][2];
#pragma unroll
            for (int i = 0; i < Gm::R; ++i)
                a0[i][0] = a0[i][1] = a1[i][0] = a1[i][1] = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < Gm::K / 4; ++j) {
                const float4 u0 = *reinterpret_cast<const float4 *>(c0 + 4 * Gm::QG * j);
                const float4 u1 = *reinterpret_cast<const float4 *>(c1 + 4 * Gm::QG * j);
#pragma unroll
                for (int i = 0; i < Gm::R; ++i) {
                    a0[i][0] = __ffma2_rn(st[i][2 * j], make_float2(u0.x, u0.y), a0[i][0]);
                    a1[i][0] = __ffma2_rn(st[i][2 * j], make_float2(u1.x, u1.y), a1[i][0]);
                    a0[i][1] = __ffma2_rn(st[i][2 * j + 1], make_float2(u0.z, u0.w), a0[i][1]);
                    a1[i][1] = __ffma2_rn(st[i][2 * j + 1], make_float2(u1.z, u1.w), a1[i][1]);
                }
            }
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                if (n == 1 && !two)
                    break;
                const int i = n == 0 ? i0 : i1;
                float p[Gm::R];
#pragma unroll
                for (int r = 0; r < Gm::R; ++r) {
                    const float2 *q2 = n == 0 ? a0[r] : a1[r];
                    p[r] = (q2[0].x + q2[0].y) + (q2[1].x + q2[1].y);
                }
                float own[Gm::NOWN];
                int oi[Gm::NOWN];                // which of the lane's rows each holds
                bool ow = true;                  // whether this lane writes them
                if constexpr (Gm::QG == 1) {
#pragma unroll
                    for (int r = 0; r < Gm::R; ++r) {
                        own[r] = p[r];
                        oi[r] = r;
                    }
                } else {
                    // groups cg and cg ^ 1 exchange halves of the rows (xor LG)
                    const bool odd = cg & 1;
                    float v[Gm::R / 2];
#pragma unroll
                    for (int k = 0; k < Gm::R / 2; ++k) {
                        const float send = odd ? p[2 * k] : p[2 * k + 1];
                        const float keep = odd ? p[2 * k + 1] : p[2 * k];
                        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, Gm::LG);
                    }
                    if constexpr (Gm::QG == 2) {
#pragma unroll
                        for (int k = 0; k < Gm::R / 2; ++k) {
                            own[k] = v[k];
                            oi[k] = 2 * k + (cg & 1);
                        }
                    } else if constexpr (Gm::R == 4) {   // four groups: second exchange
                        const bool hi = cg & 2;
                        const float send = hi ? v[0] : v[1];
                        const float keep = hi ? v[1] : v[0];
                        own[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2 * Gm::LG);
                        oi[0] = (cg & 1) + 2 * (hi ? 1 : 0);
                    } else {                     // four groups, two rows
                        own[0] = v[0] + __shfl_xor_sync(0xffffffffu, v[0], 2 * Gm::LG);
                        oi[0] = cg & 1;
                        ow = (cg & 2) == 0;
                    }
                }
                const int cn = cnt[i];
#pragma unroll
                for (int k = 0; k < Gm::NOWN; ++k) {
                    const int d = rb + oi[k] * Gm::LG;
                    if (!ow || d >= u.rows)
                        continue;
                    float y = 0.f;
                    if (cn > 0)
                        y = fmaf(wt[i], own[k], psum[i * kTile + d]) +
                            Dh * xs_at(xs, a.x_dtype, i * kXS + d);
                    st_f32(a.out, a.x_dtype,
                           (((int64_t)u.b * T + i) * H + u.h) * Dm + u.row0 + d, y);
                }
            }
        }
        __syncthreads();                 // every read of this item's buffers is done
        if (next_valid && xasync && !x_mid) {
            prefetch_x(ta, lay.xs, lay.xbytes, sm, v, 0);
            cp_async_commit();
        }
    }
    cp_async_wait_all();                 // no copy outlives the CTA
}

// ---------------------------------------------------------------- tensor-core form
//
// With bf16 B and C and dstate 64 or 128, the dense products run on the tensor cores.
// For item (b, h, dim tile) they form one matrix product: D[i][d] = sum_n C_i[n] s0[d][n]
// for the 128 node slots i (slots T .. 127 hold zero C rows) and the tile's 64 dim rows d.
// C is bf16, so it enters the MMA exactly; the committed state is split into bf16
// pieces s0 = p1 + p2 + p3 by truncation (p1 = s0 with its low 16 bits cleared, p2 the
// same of s0 - p1, p3 = s0 - p1 - p2: each difference is exact in fp32, and p3 keeps at
// most the 8 significant bits a bf16 holds, so the pieces sum to s0 exactly), and every
// product of two bf16 values is exact in the fp32 accumulator. The pieces are stacked as the rows of one B operand (64 rows each), so a
// single chain of dstate / 16 MMAs of N = 64 x pieces reads C once and leaves C p1^T,
// C p2^T and C p3^T side by side in tensor memory (128 lanes = slots, 64 fp32 columns
// per piece), summed smallest first in the epilogue. An fp16 state needs two pieces
// (11 significant bits), a bf16 state one.
//
// A CTA of 16 warps takes a share of one row's items when there are at least as many
// CTAs as rows, else a contiguous range of items. Per (row, group) the row's tables are
// built once (stage_row_tc): the path pairs and their C_i . B_j, and the nodes ranked by
// path length, node i's C row going to operand row (slot) rank(i). Per item, in order:
// the state rows (one bulk copy) and the x tile (one tensor copy, 128-byte swizzled),
// issued during the previous item, are waited for; the state rows are split into the
// pieces and the nodes' dt_eff and dA formed; thread 0 issues the MMAs and commits them
// to an mbarrier, while the producer thread starts the next item's copies and every
// thread forms its path sums: warp w takes slots 8w .. 8w + 7 with four lanes each and
// 16 dim rows per lane, so a warp's paths are about equally long, with the coefficients
// w_im dt_jm (C_i . B_jm) built on the way; then the stash's U is written. Once the MMAs
// are done, the path sums and each slot's W go through shared memory (over the pieces)
// to the epilogue thread of the slot (a warp's lanes are the TMEM lanes of its quarter),
// which forms out = W_i D + P + D_h x and writes it over its x values in the tile; one
// tensor store per tile sends it out.

constexpr int kTcThreads = 512;       // 16 warps, one CTA per SM
constexpr uint32_t kTcCols = 256;     // TMEM columns: 64 dim rows per state piece (<= 3)

// Shared-memory layout of the tensor-core form (byte offsets from a 1024-byte aligned
// base). npc state pieces; E bounds the path pairs as in TLayout.
struct TcLayout {
    int ca, sp, raw, xs, tp, xbytes, cb, pj, pi, par, cnt, off, sn, ns, wsl, da, dtv, bar, tptr,
        total;
    __host__ __device__ static int up16(int v) { return (v + 15) & ~15; }
    __host__ __device__ TcLayout(int T, int N, int es_x, int es_s, int npc, int nxb)
    {
        const int E = T * (T + 1) / 2;
        ca = 0;                               // C operand: N / 64 blocks of 128 x 128 B
        sp = ca + 128 * N * 2;                // pieces: npc x N / 64 blocks of 64 x 128 B
        // (the same bytes stage the row's B rows between items, 128 x N bf16, and hand the
        // path sums to the epilogue once an item's products are done, 32 KB)
        int spb = (npc * kTile > 128 ? npc * kTile : 128) * N * 2;
        spb = spb > 32768 ? spb : 32768;
        raw = sp + spb;                       // state rows as stored
        // x tiles: kTile * es_x / 128 blocks of tp 128-byte rows (see xt_off), each block
        // 1024-byte aligned
        xs = (raw + kTile * N * es_s + 1023) & ~1023;
        tp = (T + 7) & ~7;
        xbytes = (kTile * es_x / 128) * tp * 128;
        cb = xs + nxb * xbytes;
        pj = cb + up16(E * 4);
        pi = pj + up16(E);
        par = pi + up16(E);
        cnt = par + up16(T * 4);
        off = cnt + up16(T * 4);
        sn = off + up16((T + 1) * 4);        // node of each operand row (slot)
        ns = sn + up16(T);                    // slot of each node
        wsl = ns + up16(T);                   // W of each slot's node (128 floats)
        da = wsl + 128 * 4;                   // {dt_eff, dA} of each node (float2)
        dtv = da;
        bar = da + up16(T * 8);               // mbarriers: MMA, state rows, x tiles 0 / 1
        tptr = bar + 32;
        total = tptr + 16 + 1024;             // slack for aligning the base
    }
};

// Per-(row, group) tables of the tensor-core form: parents, path checks, C in the
// operand layout, path pairs (pj: path node, pi: node) and C_i . B_j of every pair. The
// row's B rows are fetched into the piece buffer (free between items; 16-byte chunks
// XOR-swizzled by the row) by cp.async and its C rows into registers, all at once, while
// parents and depths load and every node's path is walked. The nodes are then ranked by
// path length, and node i's C row goes to operand row (slot) ns[i] = its rank (sn[] maps
// back): the accumulator lane of a slot is its node's, and the threads that take a
// warp's 32 slots in the per-item path sums then have paths of about equal length, so
// that no warp runs many more path steps than its lanes need. The C . B products then
// read shared memory only. The staged B rows also give the stash its B: the shares of
// heads hh0 .. hh1 (indices within the group) of this CTA's items, each head's share
// being elements [T N hh / hpg, T N (hh + 1) / hpg) of the row's [T][N] block.
//
// The kernel calls it behind a barrier, so every buffer of the previous item is free.
template <int N>
__device__ void stage_row_tc(const TreeArgs &ta, const TcLayout &lay, uint8_t *sm, int b, int g,
                             bool reporter, int hh0, int hh1)
{
    constexpr int CPR = N / 8;                // 16-byte chunks per bf16 row
    constexpr int CQ = 128 * CPR / kTcThreads;    // C chunks per thread (128 operand rows)
    const DecodeArgs &a = ta.d;
    const int T = ta.T, G = a.G, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *cb = reinterpret_cast<float *>(sm + lay.cb);
    uint8_t *pj = sm + lay.pj;
    uint8_t *pi = sm + lay.pi;
    uint8_t *sn = sm + lay.sn;
    uint8_t *ns = sm + lay.ns;
    uint8_t *bst = sm + lay.sp;               // B rows of the row's nodes
    int *par = reinterpret_cast<int *>(sm + lay.par);
    int *cnt = reinterpret_cast<int *>(sm + lay.cnt);
    int *off = reinterpret_cast<int *>(sm + lay.off);
    const uint16_t *Cg = static_cast<const uint16_t *>(a.C);
    const uint16_t *Bg = static_cast<const uint16_t *>(a.B);

    uint4 creg[CQ];                           // chunk tid + q * threads: row k / CPR
#pragma unroll
    for (int q = 0; q < CQ; ++q) {
        const int k = tid + q * kTcThreads, i = k / CPR, c = k % CPR;
        creg[q] = i < T ? *reinterpret_cast<const uint4 *>(Cg + (((int64_t)b * T + i) * G + g) * N + c * 8)
                        : make_uint4(0u, 0u, 0u, 0u);
    }
    for (int k = tid; k < T * CPR; k += kTcThreads) {
        const int j = k / CPR, c = k % CPR;
        cp_async16(bst + j * (N * 2) + ((c ^ (j & 7)) << 4),
                   Bg + (((int64_t)b * T + j) * G + g) * N + c * 8);
    }
    cp_async_commit();
    int depth = 0;                            // node tid's depth (T <= 128 < threads)
    if (tid < T) {
        par[tid] = ta.parents[(int64_t)b * T + tid];
        depth = ta.depths[(int64_t)b * T + tid];
    }
    __syncthreads();
    // every node's walk: exactly depth parent steps inside [0, T), then parent -1
    if (tid < T) {
        bool ok = depth >= 0 && depth < kMaxNodes;
        int j = tid;
        for (int k = 0; ok && k < depth; ++k) {
            j = par[j];
            ok = j >= 0 && j < T;
        }
        ok = ok && par[j] == -1;
        cnt[tid] = ok ? depth + 1 : 0;
        if (!ok && reporter && a.err)
            atomicOr(a.err, SSU_FLAG_TREE);
    } else if (tid < ((T + 3) & ~3)) {
        cnt[tid] = 0x7fffffff;               // padding to a whole int4, ranked after all
    }
    __syncthreads();
    if (warp == 0) {                          // exclusive prefix sum; off[T] = all pairs
        int carry = 0;
        for (int base = 0; base < T; base += 32) {
            const int i = base + lane;
            const int v = i < T ? cnt[i] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += t;
            }
            if (i < T)
                off[i] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0)
            off[T] = carry;
    } else if (tid >= 128 && tid < 128 + T) { // rank by path length, ties by node index
        const int i = tid - 128, ci = cnt[i];
        int r = 0;
        for (int k = 0; k < T; k += 4) {
            const int4 c4 = *reinterpret_cast<const int4 *>(cnt + k);
            r += (c4.x < ci || (c4.x == ci && k < i)) + (c4.y < ci || (c4.y == ci && k + 1 < i)) +
                 (c4.z < ci || (c4.z == ci && k + 2 < i)) + (c4.w < ci || (c4.w == ci && k + 3 < i));
        }
        ns[i] = static_cast<uint8_t>(r);
        sn[r] = static_cast<uint8_t>(i);
    }
    __syncthreads();
    // C rows into their slots; the slots past T (no node) are zero
#pragma unroll
    for (int q = 0; q < CQ; ++q) {
        const int k = tid + q * kTcThreads, i = k / CPR, c = k % CPR;
        *reinterpret_cast<uint4 *>(sm + lay.ca + sw128_off(i < T ? ns[i] : i, c, 128 * 128)) =
            creg[q];
    }
    if (tid < T) {
        const int c = cnt[tid], o = off[tid];
        int j = tid;
        for (int k = 0; k < c; ++k) {
            pj[o + k] = static_cast<uint8_t>(j);
            pi[o + k] = static_cast<uint8_t>(tid);
            j = par[j];
        }
    }
    cp_async_wait_all();                      // B rows landed
    __syncthreads();
    const int total = off[T];
    for (int p = tid; p < total; p += kTcThreads) {
        const int i = pi[p], j = pj[p], si = ns[i];
        const uint8_t *brow = bst + j * (N * 2);
        float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < CPR; ++c) {
            const uint4 cv = *reinterpret_cast<const uint4 *>(sm + lay.ca + sw128_off(si, c, 128 * 128));
            const uint4 bv = *reinterpret_cast<const uint4 *>(brow + ((c ^ (j & 7)) << 4));
            const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)       // a bf16 pair widens to floats by shift and mask
                s2[q & 1] = __ffma2_rn(
                    make_float2(__uint_as_float(cw[q] << 16), __uint_as_float(cw[q] & 0xFFFF0000u)),
                    make_float2(__uint_as_float(bw[q] << 16), __uint_as_float(bw[q] & 0xFFFF0000u)),
                    s2[q & 1]);
        }
        cb[p] = (s2[0].x + s2[0].y) + (s2[1].x + s2[1].y);
    }
    if (hh0 <= hh1) {                         // stash B: this CTA's heads' shares
        const int hpg = a.H / G, total = T * N;
        const int e0 = total * hh0 / hpg, e1 = total * (hh1 + 1) / hpg;
        const int64_t rbase = ((int64_t)b * T * G + g) * N;     // node 0 of the row
        for (int e = e0 + tid; e < e1; e += kTcThreads) {
            const int j = e / N, n = e - j * N;
            const uint16_t bits = *reinterpret_cast<const uint16_t *>(
                bst + j * (N * 2) + (((n >> 3) ^ (j & 7)) << 4) + (n & 7) * 2);
            ta.st_B[rbase + (int64_t)j * G * N + n] = __uint_as_float((uint32_t)bits << 16);
        }
    }
}

// Number of bf16 pieces that carry a state element exactly (fp32: to within 2^-24 of it).
template <typename S> struct Pieces { static constexpr int n = 3; };
template <> struct Pieces<__half> { static constexpr int n = 2; };
template <> struct Pieces<__nv_bfloat16> { static constexpr int n = 1; };

// The item's state rows (raw staging, row-major) split into bf16 pieces in the operand
// layout; rows >= rows are zero.
template <typename S, int N>
__device__ void split_state(const TcLayout &lay, uint8_t *sm, int rows)
{
    constexpr int CPR = N / 8, NPC = Pieces<S>::n;
    for (int e = threadIdx.x; e < kTile * CPR; e += kTcThreads) {
        const int r = e / CPR, c = e % CPR;
        float f[8];
        if (r < rows) {
            const uint8_t *src = sm + lay.raw + (r * N + c * 8) * (int)sizeof(S);
            if constexpr (sizeof(S) == 4) {
                Vec16<float>::unpack(*reinterpret_cast<const uint4 *>(src), f);
                Vec16<float>::unpack(*reinterpret_cast<const uint4 *>(src + 16), f + 4);
            } else {
                Vec16<S>::unpack(*reinterpret_cast<const uint4 *>(src), f);
            }
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q)
                f[q] = 0.f;
        }
#pragma unroll
        for (int p = 0; p < NPC; ++p) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                // the piece is the value with the low 16 bits cleared (bf16 truncation); two
                // pieces' high halves pack into one word by a byte permute
                const uint32_t u0 = __float_as_uint(f[2 * q]), u1 = __float_as_uint(f[2 * q + 1]);
                w[q] = __byte_perm(u0, u1, 0x7632);
                if (p + 1 < NPC) {             // the rest, exact: it is f's low mantissa bits
                    f[2 * q] -= __uint_as_float(u0 & 0xFFFF0000u);
                    f[2 * q + 1] -= __uint_as_float(u1 & 0xFFFF0000u);
                }
            }
            *reinterpret_cast<uint4 *>(sm + lay.sp + sw128_off(p * kTile + r, c, NPC * kTile * 128)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// Bulk (TMA) copies of an item's inputs; each buffer completes on its own mbarrier, armed
// by one thread with the whole byte count. The state rows are one contiguous block (at most
// four copies by the leader).
template <typename S, int N>
__device__ __forceinline__ void bulk_raw(const TreeArgs &ta, const TcLayout &lay, uint8_t *sm,
                                         const Item &u, uint64_t *bar, bool leader,
                                         uint32_t extra)
{
    if (!leader)
        return;
    const DecodeArgs &a = ta.d;
    const char *src = static_cast<const char *>(a.state) +
                      ((int64_t)u.slot * a.slot_stride + ((int64_t)u.h * a.Dm + u.row0) * N) *
                          (int64_t)sizeof(S);
    const uint32_t bytes = (uint32_t)(u.rows * N * (int)sizeof(S));
    const uint32_t part = ((bytes + 3) / 4 + 15) & ~15u;
    mbar_arrive_expect_tx(bar, bytes + extra);
    for (uint32_t o = 0; o < bytes; o += part)
        bulk_load(sm + lay.raw + o, src + o, bytes - o < part ? bytes - o : part, bar);
}

// Byte offset in an x tile of the 16-byte chunk holding dims d .. d + 16 / es - 1 of node
// i (d a multiple of 16 / es). The tile is kTile * es / 128 blocks of tp rows of 128 bytes
// (64 / es dims), and the chunks of row i are XOR-swizzled by i % 8: the layout the tensor
// copies' 128-byte swizzle gives a 1024-byte aligned box. Lanes reading the same chunk of
// different rows (the path sums) or their own rows (the epilogue) thereby spread over the
// banks.
template <typename X>
__device__ __forceinline__ int xt_off(int i, int d, int tp)
{
    constexpr int es = (int)sizeof(X), per = 128 / es;
    const int c = (d % per) * es / 16;
    return (d / per) * (tp * 128) + i * 128 + ((c ^ (i & 7)) << 4);
}

// Element d of node i of an x tile, widened.
template <typename X>
__device__ __forceinline__ float xt_at(const uint8_t *xs, int i, int d, int tp)
{
    constexpr int es = (int)sizeof(X), per16 = 16 / es;
    const uint8_t *p = xs + xt_off<X>(i, d - d % per16, tp) + (d % per16) * es;
    if constexpr (es == 4)
        return *reinterpret_cast<const float *>(p);
    else
        return bits_f32(*reinterpret_cast<const uint16_t *>(p),
                        std::is_same<X, __half>::value ? SSU_F16 : SSU_BF16);
}

// The x tile of item u by one tensor copy per 128-byte block (thread `issuer` arms the
// barrier and issues them): rows 0 .. T - 1 of the tile, dims past Dm read as zero.
template <typename X>
__device__ __forceinline__ void tma_x(const TreeArgs &ta, const CUtensorMap *xmap, uint8_t *xs,
                                      const Item &u, uint64_t *bar, uint32_t extra, int tp)
{
    constexpr int nblk = kTile * (int)sizeof(X) / 128, per = 128 / (int)sizeof(X);
    mbar_arrive_expect_tx(bar, (uint32_t)(nblk * ta.T * 128) + extra);
#pragma unroll
    for (int q = 0; q < nblk; ++q)
        tma_load_rows(xs + q * tp * 128, xmap, u.row0 + q * per, u.h, u.b * ta.T, bar);
}

// The x tile of item u with plain loads, in the same layout (x rows not 16-byte aligned,
// or too short for a tensor copy): dims >= u.rows are 0.
template <typename X>
__device__ void stage_x_tc(const TreeArgs &ta, uint8_t *xs, const Item &u, int tp)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, Dm = a.Dm;
    constexpr int per16 = 16 / (int)sizeof(X);            // dims per 16-byte chunk
    for (int e = threadIdx.x; e < T * (kTile / per16); e += kTcThreads) {
        const int i = e / (kTile / per16), d = per16 * (e % (kTile / per16));
        const int64_t src = (((int64_t)u.b * T + i) * H + u.h) * Dm + u.row0 + d;
        float f[per16];
#pragma unroll
        for (int q = 0; q < per16; ++q)
            f[q] = d + q < u.rows ? ld_f32(a.x, a.x_dtype, src + q) : 0.f;
        *reinterpret_cast<uint4 *>(xs + xt_off<X>(i, d, tp)) = Vec16<X>::pack(f);
    }
}

// 16 consecutive x values of node i from dim row d0 (a multiple of 16) of an x tile, and
// the same positions overwritten (rounded to X).
template <typename X>
__device__ __forceinline__ void x_seg16(const uint8_t *xs, int i, int d0, int tp, float (&f)[16])
{
    constexpr int per = 16 / (int)sizeof(X);
#pragma unroll
    for (int q = 0; q < 16 / per; ++q)
        Vec16<X>::unpack(*reinterpret_cast<const uint4 *>(xs + xt_off<X>(i, d0 + per * q, tp)),
                         f + per * q);
}

// The same 16 values as 8 pairs (dims d0 + 2q, d0 + 2q + 1), for packed arithmetic.
template <typename X>
__device__ __forceinline__ void x_pairs16(const uint8_t *xs, int i, int d0, int tp, float2 (&f)[8])
{
    if constexpr (sizeof(X) == 4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = *reinterpret_cast<const float4 *>(xs + xt_off<X>(i, d0 + 4 * q, tp));
            f[2 * q] = make_float2(v.x, v.y);
            f[2 * q + 1] = make_float2(v.z, v.w);
        }
    } else {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint4 v = *reinterpret_cast<const uint4 *>(xs + xt_off<X>(i, d0 + 8 * q, tp));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if constexpr (std::is_same<X, __nv_bfloat16>::value) {
                    f[4 * q + k] = make_float2(__uint_as_float(w[k] << 16),
                                               __uint_as_float(w[k] & 0xFFFF0000u));
                } else {
                    __half2 h;
                    memcpy(&h, &w[k], 4);
                    f[4 * q + k] = __half22float2(h);
                }
            }
        }
    }
}

template <typename X>
__device__ __forceinline__ void put_seg16(uint8_t *xs, int i, int d0, int tp, const float (&y)[16])
{
    constexpr int per = 16 / (int)sizeof(X);
#pragma unroll
    for (int q = 0; q < 16 / per; ++q)
        *reinterpret_cast<uint4 *>(xs + xt_off<X>(i, d0 + per * q, tp)) = Vec16<X>::pack(y + per * q);
}

// U of the item (x widened to fp32): 16 bytes of the tile per task, 16-byte stores; thread
// t of the nt taking part.
template <typename X>
__device__ void stash_u_tc(const TreeArgs &ta, const Item &u, const uint8_t *xs, int tp, int t,
                           int nt)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, Dm = a.Dm;
    constexpr int per = 16 / (int)sizeof(X);              // x values per task
    if ((Dm & 3) == 0 && (reinterpret_cast<uintptr_t>(ta.st_U) & 15) == 0) {
        for (int e = t; e < T * (kTile / per); e += nt) {
            const int i = e / (kTile / per), d = per * (e % (kTile / per));
            if (d < u.rows) {
                float f[per];
                Vec16<X>::unpack(*reinterpret_cast<const uint4 *>(xs + xt_off<X>(i, d, tp)), f);
                float *dst = ta.st_U + (((int64_t)u.b * T + i) * H + u.h) * Dm + u.row0 + d;
#pragma unroll
                for (int q = 0; q < per / 4; ++q)
                    if (d + 4 * q < u.rows)
                        *reinterpret_cast<float4 *>(dst + 4 * q) =
                            make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
            }
        }
    } else {
        for (int e = t; e < T * kTile; e += nt) {
            const int i = e / kTile, d = e % kTile;
            if (d < u.rows)
                ta.st_U[(((int64_t)u.b * T + i) * H + u.h) * Dm + u.row0 + d] =
                    xt_at<X>(xs, i, d, tp);
        }
    }
}

// dt_eff and dA of every node for the item's head (node threadIdx.x, from its prefetched
// dt) into shared memory as {dt_eff, dA} pairs, and into the stash once per (row, head).
__device__ __forceinline__ void node_values_tc(const TreeArgs &ta, float2 *sdtA, const Item &u,
                                               float dt_mine, const HeadVals &hv)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, tid = threadIdx.x;
    if (tid < T) {
        const int64_t bi = (int64_t)u.b * T + tid;
        const float v = dt_mine + hv.bias;
        const float dte = a.softplus ? softplus_f(v) : v;
        const float dA = expf(hv.A * dte);
        sdtA[tid] = make_float2(dte, dA);
        if (u.dtile == 0) {
            ta.st_dA[bi * a.H + u.h] = dA;
            ta.st_dt[bi * a.H + u.h] = dte;
        }
    }
}

// Items of this CTA. With at least as many CTAs as rows, every CTA takes a share of one
// row's items (each CTA then builds one row's tables); otherwise contiguous ranges.
__device__ __forceinline__ void cta_range(int64_t nitems, int64_t per_row, int rows,
                                          int64_t &first, int64_t &last)
{
    const int64_t c = blockIdx.x, grid = gridDim.x;
    if (grid >= rows && rows > 0) {
        const int64_t r = c * rows / grid;
        const int64_t c0 = (r * grid + rows - 1) / rows, c1 = ((r + 1) * grid + rows - 1) / rows;
        first = r * per_row + per_row * (c - c0) / (c1 - c0);
        last = r * per_row + per_row * (c - c0 + 1) / (c1 - c0);
    } else {
        first = nitems * c / grid;
        last = nitems * (c + 1) / grid;
    }
}

// xtma / otma: the x tiles come in and the outputs go out by tensor copies (tensor maps
// xmap / omap over x and out); otherwise the x tiles are staged with plain loads and each
// thread stores its own outputs.
template <typename S, typename X, int N>
__global__ void __launch_bounds__(kTcThreads, 1)
ssu_ddtree_tc_kernel(const __grid_constant__ TreeArgs ta, const __grid_constant__ CUtensorMap xmap,
                     const __grid_constant__ CUtensorMap omap, const int dtiles,
                     const int64_t nitems, const int nxb, const int xtma, const int otma)
{
    constexpr int NPC = Pieces<S>::n;
    constexpr int es_x = (int)sizeof(X);
    constexpr int nblk = kTile * es_x / 128, per_blk = 128 / es_x;   // x tile blocks, dims each
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, NPC * kTile);
    // the thread that issues every copy of the items' inputs and every output store: lane 0
    // of warp 1, whose path-sum slots have short paths (as have warp 0's: thread 0 issues
    // the MMAs)
    constexpr int kProducer = 32;
    extern __shared__ __align__(16) uint8_t sm_dyn[];
    uint8_t *sm = sm_dyn + ((1024 - (smem_u32(sm_dyn) & 1023)) & 1023);
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, Dm = a.Dm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool producer = tid == kProducer;
    const TcLayout lay(T, N, es_x, (int)sizeof(S), NPC, nxb);
    const int tp = lay.tp;
    const float *cb = reinterpret_cast<const float *>(sm + lay.cb);
    const uint8_t *pj = sm + lay.pj;
    const int *cnt = reinterpret_cast<const int *>(sm + lay.cnt);
    const int *off = reinterpret_cast<const int *>(sm + lay.off);
    const uint8_t *sn = sm + lay.sn;
    float2 *sdtA = reinterpret_cast<float2 *>(sm + lay.da);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + lay.bar);     // MMA completion
    uint64_t *sbar = bar + 1;                                         // state rows landed
    uint64_t *xbar = bar + 2;                                         // x tile 0 / 1 landed
    uint32_t *tptr = reinterpret_cast<uint32_t *>(sm + lay.tptr);

    if (warp == 0)
        tmem_alloc(tptr, kTcCols);
    if (tid == 0) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            mbar_init(bar + k, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tptr;
    // this thread's slot (TMEM lane; its node is sn[ni]) and its 16 dim rows (TMEM columns)
    const int ni = 32 * (warp & 3) + lane, d0 = 16 * (warp >> 2);
    // Its path sums: slot pslot (of warp w's 8 slots 8w .. 8w + 7, four lanes each) over
    // dim rows pd0 .. pd0 + 15. The slots are ranked by path length, so the paths of a
    // warp's slots are about equally long, and the four warps of a scheduler (w, w + 4,
    // w + 8, w + 12) take slot groups from every quarter of the ranking. The sums reach the
    // slot's epilogue thread through shared memory.
    const int pslot = 8 * warp + (lane >> 2), pd0 = 16 * (lane & 3);
    const uint32_t taddr = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)d0;
    uint32_t phase = 0;                  // parity of the MMA barrier's next phase
    bool mma_out = false;                // an MMA wait gave up (its phase is still awaited)
    // copies in flight (uniform): state rows, x tiles by buffer bit; parities likewise
    uint32_t s_out = 0, x_out = 0, sph = 0, xph = 0;

    // with two x buffers the next item's tile is fetched while this one computes
    const bool x_mid = xtma && nxb == 2;
    int64_t first, last;
    cta_range(nitems, nitems / a.active, a.active, first, last);
    auto xbuf_of = [&](int64_t it) { return nxb == 2 ? (int)((it - first) & 1) : 0; };
    // the state block of item w (the raw staging must be free)
    auto issue_s = [&](const Item &w, int64_t wit) {
        bulk_raw<S, N>(ta, lay, sm, w, sbar, producer,
                       fault_tx(kFaultTreeState, -1, (int)(wit - first)));
        s_out = 1;
    };
    // the x tile of item w into its buffer (no thread may still read that buffer; the
    // producer first waits for its own output stores to have read it)
    auto issue_x = [&](const Item &w, int64_t wit) {
        const int xb = xbuf_of(wit);
        if (producer) {
            bulk_wait_read_all();
            tma_x<X>(ta, &xmap, sm + lay.xs + xb * lay.xbytes, w, xbar + xb,
                     fault_tx(kFaultTreeX, -1, (int)(wit - first)), tp);
        }
        x_out |= 1u << xb;
    };
    Item u = item_at(ta, first < last ? first : 0, dtiles);
    int nslot = row_slot(ta, u.b + 1);   // slot of the row after u's
    float dt_next = 0.f;                 // node tid's dt and the head's scalars, next item
    HeadVals hv_next = {0.f, 0.f, 0.f};
    if (first < last && u.valid(a.P)) {
        issue_s(u, first);
        if (xtma)
            issue_x(u, first);
        dt_next = dt_of(ta, u);
        hv_next = head_vals(a, u.h);
    }
    int cur_b = -1, cur_g = -1;
    Item v = u;
    for (int64_t it = first; it < last; ++it, u = v) {
        const bool has_next = it + 1 < last;
        if (has_next)
            v = item_after_pf(ta, u, dtiles, nslot);
        const bool next_valid = has_next && v.valid(a.P);
        if (!u.valid(a.P)) {
            if (u.slot < 0) {            // padding row: zero outputs at every node
                for (int e = tid; e < T * kTile; e += kTcThreads) {
                    const int i = e / kTile, dd = e % kTile;
                    if (dd < u.rows)
                        st_f32(a.out, a.x_dtype,
                               (((int64_t)u.b * T + i) * H + u.h) * Dm + u.row0 + dd, 0.f);
                }
            } else if (u.h == 0 && u.dtile == 0 && tid == 0 && a.err) {
                atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
            }
            if (next_valid) {            // this item used no buffer: start the next one
                issue_s(v, it + 1);
                if (xtma)
                    issue_x(v, it + 1);
                dt_next = dt_of(ta, v);
                hv_next = head_vals(a, v.h);
            }
            continue;
        }
        // (every thread passed the previous item's closing barrier, or its epilogue barrier
        // and the next one below)
        uint8_t *xs = sm + lay.xs + xbuf_of(it) * lay.xbytes;
        if (u.b != cur_b || u.g != cur_g) {
            // heads of (u.b, u.g) whose dim tile 0 lies in this CTA's range: their B stash
            const int hpg = H / a.G;
            const int64_t rs = (int64_t)u.b * H * dtiles;              // the row's item 0
            const int64_t i0 = (first > rs ? first : rs) - rs;
            const int64_t i1 = (last < rs + (int64_t)H * dtiles ? last : rs + (int64_t)H * dtiles) - rs;
            const int hlo = max((int)((i0 + dtiles - 1) / dtiles), u.g * hpg);
            const int hhi = min((int)((i1 - 1) / dtiles), (u.g + 1) * hpg - 1);
            __syncthreads();             // the previous item's epilogue is done with its buffers
            stage_row_tc<N>(ta, lay, sm, u.b, u.g, u.h == 0 && u.dtile == 0, hlo - u.g * hpg,
                            hhi - u.g * hpg);
            cur_b = u.b;
            cur_g = u.g;
        }
        if (!xtma) {
            if (producer)
                bulk_wait_read_all();    // an earlier output store has read this buffer
            __syncthreads();
            stage_x_tc<X>(ta, xs, u, tp);
        }
        // a copy counts as landed (its in-flight bit cleared) only once its wait succeeded,
        // so that after a give-up the final drain waits for it again
        bool landed = true;
        if (s_out) {
            if (mbar_wait(sbar, sph)) {
                sph ^= 1u;
                s_out = 0;
            } else {
                landed = false;
            }
        }
        const int xb = xbuf_of(it);
        if ((x_out >> xb) & 1u) {
            if (mbar_wait(xbar + xb, (xph >> xb) & 1u)) {
                xph ^= 1u << xb;
                x_out &= ~(1u << xb);
            } else {
                landed = false;
            }
        }
        if (__syncthreads_or(!landed)) { // state rows and x tile have landed
            if (tid == 0 && a.err)
                atomicOr(a.err, SSU_FLAG_TIMEOUT);
            break;
        }
        const HeadVals hv = hv_next;
        split_state<S, N>(lay, sm, u.rows);
        fence_async_smem();              // operands visible to the tensor cores
        node_values_tc(ta, sdtA, u, dt_next, hv);
        __syncthreads();
        if (tid == 0 && !fault_tx(kFaultTreeMma, -1, (int)(it - first))) {
            tc_fence_after();
            const uint32_t base = smem_u32(sm);
            uint32_t acc = 0;
#pragma unroll
            for (int kb = 0; kb < N / 64; ++kb)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = desc_k_sw128(base + lay.ca + kb * 16384 + kk * 32);
                    const uint64_t bd = desc_k_sw128(base + lay.sp + kb * (NPC * kTile * 128) +
                                                     kk * 32);
                    tc_mma_bf16(tmem, ad, bd, kIdesc, acc);
                    acc = 1;
                }
            tc_commit(bar);
        }
        if (next_valid) {
            issue_s(v, it + 1);          // the raw staging was consumed by the split
            // Every thread has finished the previous item, so the other x buffer (the
            // previous item's) is free once the producer's store of its outputs has read
            // it: one tensor copy brings the next item's tile there while this one computes.
            if (x_mid)
                issue_x(v, it + 1);
            dt_next = dt_of(ta, v);
            hv_next = head_vals(a, v.h);
        }

        // path sums of slot pslot's node over rows pd0 .. pd0 + 15 while the MMAs run
        float2 ps[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            ps[e] = make_float2(0.f, 0.f);
        float wi = 1.f;
        {
            const int pnode = pslot < T ? sn[pslot] : 0;
            const int cn = pslot < T ? cnt[pnode] : 0, o = off[pnode];
            for (int k = 0; k < cn; ++k) {
                const int j = pj[o + k];
                const float2 tA = sdtA[j];                // {dt_eff, dA}
                const float cf = wi * tA.x * cb[o + k];
                wi *= tA.y;
                float2 xv[8];
                x_pairs16<X>(xs, j, pd0, tp, xv);
                const float2 c2 = make_float2(cf, cf);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    ps[e] = __ffma2_rn(c2, xv[e], ps[e]);
            }
        }
        stash_u_tc<X>(ta, u, xs, tp, tid, kTcThreads);
        const bool ok = mbar_wait(bar, phase);
        if (__syncthreads_or(!ok)) {     // the MMAs never completed: give up on the launch
            if (tid == 0 && a.err)
                atomicOr(a.err, SSU_FLAG_TIMEOUT);
            mma_out = true;
            break;
        }
        phase ^= 1u;
        tc_fence_after();
        // hand over the path sums (the piece buffer is free: the products are done): slot s
        // takes 256 bytes, its 16-byte chunk c (dims 4c .. 4c + 3) at position c ^ (s % 16),
        // so that the epilogue's lanes (consecutive slots, the same chunks) spread over the
        // banks; and W of every slot's node
        uint8_t *pex = sm + lay.sp;
        float *wsl = reinterpret_cast<float *>(sm + lay.wsl);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            *reinterpret_cast<float4 *>(pex + pslot * 256 + (((pd0 / 4 + c) ^ (pslot & 15)) << 4)) =
                make_float4(ps[2 * c].x, ps[2 * c].y, ps[2 * c + 1].x, ps[2 * c + 1].y);
        if ((lane & 3) == 0)
            wsl[pslot] = wi;
        __syncthreads();
        float pv[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float4 v4 =
                *reinterpret_cast<const float4 *>(pex + ni * 256 + (((d0 / 4 + c) ^ (ni & 15)) << 4));
            pv[4 * c] = v4.x;
            pv[4 * c + 1] = v4.y;
            pv[4 * c + 2] = v4.z;
            pv[4 * c + 3] = v4.w;
        }
        const float wn = wsl[ni];
        const int node = ni < T ? sn[ni] : 0;
        float dv[16];                    // the pieces' products, smallest first
        tmem_ld16(taddr + (uint32_t)((NPC - 1) * kTile), dv);
#pragma unroll
        for (int p = NPC - 2; p >= 0; --p) {
            float dp[16];
            tmem_ld16(taddr + (uint32_t)(p * kTile), dp);
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
                const float2 t2 = __fadd2_rn(make_float2(dv[e], dv[e + 1]), make_float2(dp[e], dp[e + 1]));
                dv[e] = t2.x;
                dv[e + 1] = t2.y;
            }
        }
        const bool mine = ni < T && d0 < u.rows;
        float y[16];
        if (mine) {
            float2 xv[8];
            x_pairs16<X>(xs, node, d0, tp, xv);
            const bool live = cnt[node] > 0;
            const float2 w2 = make_float2(wn, wn), D2 = make_float2(hv.D, hv.D);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float2 y2 = __ffma2_rn(D2, xv[e], __ffma2_rn(w2, make_float2(dv[2 * e], dv[2 * e + 1]),
                                                                  make_float2(pv[2 * e], pv[2 * e + 1])));
                y[2 * e] = live ? y2.x : 0.f;
                y[2 * e + 1] = live ? y2.y : 0.f;
            }
        }
        tc_fence_before();
        if (otma) {
            // the outputs over the x values in the tile, then one tensor store per block
            // (dims past Dm are not written)
            if (mine)
                put_seg16<X>(xs, node, d0, tp, y);
            fence_async_smem();          // these writes visible to the store
            __syncthreads();             // the tile holds every output of the item
            if (producer) {
#pragma unroll
                for (int q = 0; q < nblk; ++q)
                    tma_store_rows(&omap, xs + q * tp * 128, u.row0 + q * per_blk, u.h, u.b * T);
                bulk_commit_group();
            }
        } else if (mine) {
            const int64_t base = (((int64_t)u.b * T + node) * H + u.h) * Dm + u.row0 + d0;
#pragma unroll
            for (int e = 0; e < 16; ++e)
                if (d0 + e < u.rows)
                    st_f32(a.out, a.x_dtype, base + e, y[e]);
        }
        // Every read of this item's buffers done. Not needed when the x tile is double-
        // buffered and the next item is valid: until the next item's first barrier (its
        // row staging starts with one) a thread writes nothing this item still reads, and
        // this item's x tile is refilled only after that barrier (by the producer, once its
        // store has read the tile). The parity cases with several items per CTA crossing a
        // (row, group) change (tests/test_gpu_ddtree.py, many rows over groups and dim
        // tiles) run this path.
        if (!(x_mid && next_valid))
            __syncthreads();
        if (next_valid && xtma && !x_mid)
            issue_x(v, it + 1);
    }
    // No copy outlives the CTA and no MMA outlives its TMEM: after a give-up every copy
    // still marked in flight and the awaited MMA phase are waited for once more (bounded).
    // Should one of these waits run out as well (never expected), its copy may still
    // write this CTA's shared memory, or its MMAs the released TMEM, after the CTA ends.
    if (s_out)
        mbar_wait(sbar, sph);
    for (int k = 0; k < 2; ++k)
        if ((x_out >> k) & 1u)
            mbar_wait(xbar + k, (xph >> k) & 1u);
    if (mma_out)
        mbar_wait(bar, phase);
    if (producer)
        bulk_wait_all();                 // the output stores are complete
    cp_async_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, kTcCols);
}

// The tensor-core form when it applies (bf16 B and C with 16-byte aligned C, dstate 64 or
// 128, layout within the shared-memory limit); -1 otherwise. x and out take tensor copies
// when their rows allow (16-byte aligned, at least 128 bytes of dims).
template <typename S, typename X, int N>
int launch_tc_x(const TreeArgs &a, cudaStream_t stream, int64_t nitems, int dtiles)
{
    constexpr int es_x = (int)sizeof(X);
    int nxb = 2;
    TcLayout lay(a.T, N, es_x, (int)sizeof(S), Pieces<S>::n, nxb);
    if (lay.total > kSmemMax) {
        nxb = 1;
        lay = TcLayout(a.T, N, es_x, (int)sizeof(S), Pieces<S>::n, nxb);
    }
    if (lay.total > kSmemMax)
        return -1;
    const KernelFacts *f = kernel_facts<ssu_ddtree_tc_kernel<S, X, N>>(kTcThreads, kSmemMax);
    if (!f || f->status != SSU_OK)
        return SSU_ERR_CUDA;
    CUtensorMap xmap, omap;
    memset(&xmap, 0, sizeof xmap);
    memset(&omap, 0, sizeof omap);
    const int64_t rows = (int64_t)a.d.active * a.T;    // the rows the items touch
    const int xtma = encode_rows_map(&xmap, a.d.x, a.d.x_dtype, a.d.Dm, a.d.H, rows, a.T);
    const int otma = encode_rows_map(&omap, a.d.out, a.d.x_dtype, a.d.Dm, a.d.H, rows, a.T);
    const int64_t grid = nitems < f->sms ? nitems : f->sms;
    return launch_kernel(ssu_ddtree_tc_kernel<S, X, N>, (unsigned)grid, kTcThreads, lay.total,
                         stream, a, xmap, omap, dtiles, nitems, nxb, xtma, otma);
}

template <typename S, int N>
int launch_tc(const TreeArgs &a, cudaStream_t stream, int64_t nitems, int dtiles)
{
    if constexpr (N != 64 && N != 128) {
        return -1;
    } else {
        if (a.d.bc_dtype != SSU_BF16 || (reinterpret_cast<uintptr_t>(a.d.C) & 15) != 0)
            return -1;
        switch (a.d.x_dtype) {
        case SSU_F32: return launch_tc_x<S, float, N>(a, stream, nitems, dtiles);
        case SSU_F16: return launch_tc_x<S, __half, N>(a, stream, nitems, dtiles);
        default: return launch_tc_x<S, __nv_bfloat16, N>(a, stream, nitems, dtiles);
        }
    }
}

template <typename S, int N>
int launch_n(const TreeArgs &a, cudaStream_t stream)
{
    using Gm = TGeo<N>;
    const int dtiles = (a.d.Dm + kTile - 1) / kTile;
    const int64_t nitems = (int64_t)a.d.active * a.d.H * dtiles;
    if (nitems == 0 || a.T == 0)
        return SSU_OK;
    const int es_x = a.d.x_dtype == SSU_F32 ? 4 : 2;
    // x rows go through cp.async when every 16-byte chunk of a tile row is aligned
    const int xasync = (reinterpret_cast<uintptr_t>(a.d.x) & 15) == 0 &&
                       ((int64_t)a.d.Dm * es_x) % 16 == 0;
    const int tc = launch_tc<S, N>(a, stream, nitems, dtiles);
    if (tc >= 0)
        return tc;
    int nxb = 2;
    TLayout lay(a.T, N, es_x, (int)sizeof(S), nxb);
    if (lay.total > kSmemMax) {
        nxb = 1;
        lay = TLayout(a.T, N, es_x, (int)sizeof(S), nxb);
    }
    if (lay.total > kSmemMax)
        return SSU_ERR_UNSUPPORTED;
    const KernelFacts *f = kernel_facts<ssu_ddtree_kernel<S, N>>(kThreads, kSmemMax);
    if (!f || f->status != SSU_OK)
        return SSU_ERR_CUDA;
    const int64_t grid = nitems < f->sms ? nitems : f->sms;
    return launch_kernel(ssu_ddtree_kernel<S, N>, (unsigned)grid, kThreads, lay.total, stream, a,
                         dtiles, nitems, nxb, xasync);
}

template <typename S>
int launch_s(const TreeArgs &a, cudaStream_t s)
{
    switch (a.d.N) {
    case 8: return launch_n<S, 8>(a, s);
    case 16: return launch_n<S, 16>(a, s);
    case 32: return launch_n<S, 32>(a, s);
    case 64: return launch_n<S, 64>(a, s);
    case 128: return launch_n<S, 128>(a, s);
    case 256: return launch_n<S, 256>(a, s);
    default: return SSU_ERR_UNSUPPORTED;
    }
}

}  // namespace

#ifdef SSU_WAIT_TEST
SSU_WAIT_FAULT_SETTER(wait_fault_set_ddtree)
#endif

int launch_ddtree(const TreeArgs &a, int state_dtype, cudaStream_t s)
{
    switch (state_dtype) {
    case SSU_F32: return launch_s<float>(a, s);
    case SSU_F16: return launch_s<__half>(a, s);
    case SSU_BF16: return launch_s<__nv_bfloat16>(a, s);
    default: return SSU_ERR_DTYPE;
    }
}

}  // namespace ssu
