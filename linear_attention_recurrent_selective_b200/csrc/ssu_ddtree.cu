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
#include "ssu_async.cuh"
#include "ssu_common.cuh"
#include "ssu_tc.cuh"

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

// The item after u in row-major order; the slot index is loaded again only when the row
// changes.
__device__ __forceinline__ Item item_after(const TreeArgs &ta, const Item &u, int dtiles)
{
    const DecodeArgs &a = ta.d;
    Item v = u;
    if (++v.dtile == dtiles) {
        v.dtile = 0;
        if (++v.h == a.H) {
            v.h = 0;
            ++v.b;
            v.slot = a.idx ? a.idx[v.b] : v.b;
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
// for the 128 node slots i (rows T .. 127 of C are zero) and the tile's 64 dim rows d.
// C is bf16, so it enters the MMA exactly; the committed state is split into bf16
// pieces s0 = p1 + p2 + p3 (p1 = bf16(s0), p2 = bf16(s0 - p1), p3 = bf16(s0 - p1 - p2);
// each difference is exact in fp32, and the three pieces carry 24 significant bits, the
// fp32 significand), every product of two bf16 values is exact in the fp32 accumulator,
// and D = C p3^T + C p2^T + C p1^T accumulates in fp32. An fp16 state needs two pieces
// (11 significant bits), a bf16 state one. D lives in tensor memory: 128 lanes (node
// slots) x 64 fp32 columns (dim rows).
//
// A CTA of 16 warps takes a share of one row's items when there are at least as many
// CTAs as rows, else a contiguous range of items. Per item, in order: the state rows and
// the x tile (bulk copies issued during the previous item, each buffer on its own
// mbarrier) are waited for; the state rows are split into the pieces in the
// 128-byte-swizzled operand layout and the nodes' dt_eff and dA formed; thread 0 issues
// the MMAs (pieces x dstate / 16 of them) and commits them to an mbarrier, while the
// other threads start the next item's copies (the x rows one per thread), write the
// stash's U and form the path sums, a thread per node and 16 dim rows (thread t: node
// 32 (warp % 4) + lane, rows 16 (warp / 4) ..), with the path coefficients
// w_im dt_jm (C_i . B_jm) built on the way; then each thread reads its node's 16
// accumulator columns from tensor memory (a warp's lanes are the TMEM lanes of its
// quarter), forms out = W_i D + P + D_h x and writes it over its x values in the tile,
// which then goes out as whole 16-byte-aligned rows. Per (row, group) the row's tables
// are built once in the CTA (see stage_row_tc): C in the operand layout, the path pairs
// and their C_i . B_j from the row's B rows staged in shared memory, which also give
// the stash its B.

constexpr int kTcThreads = 512;       // 16 warps, one CTA per SM
constexpr uint32_t kTcCols = 64;      // TMEM columns: the 64 dim rows of a tile

// Shared-memory layout of the tensor-core form (byte offsets from a 1024-byte aligned
// base). npc state pieces; E bounds the path pairs as in TLayout.
struct TcLayout {
    int ca, sp, raw, xs, xbytes, cb, pj, pi, par, cnt, off, da, dtv, bar, tptr, total;
    __host__ __device__ static int up16(int v) { return (v + 15) & ~15; }
    __host__ __device__ TcLayout(int T, int N, int es_x, int es_s, int npc, int nxb)
    {
        const int E = T * (T + 1) / 2;
        ca = 0;                               // C operand: N / 64 blocks of 128 x 128 B
        sp = ca + 128 * N * 2;                // pieces: npc x N / 64 blocks of 64 x 128 B
        // (between items the same bytes stage the row's B rows: 128 x N bf16)
        raw = sp + (npc * kTile > 128 ? npc * kTile : 128) * N * 2;   // state rows as stored
        xs = raw + up16(kTile * N * es_s);
        xbytes = up16(T * kXS * es_x);
        cb = xs + nxb * xbytes;
        pj = cb + up16(E * 4);
        pi = pj + up16(E);
        par = pi + up16(E);
        cnt = par + up16(T * 4);
        off = cnt + up16(T * 4);
        da = off + up16((T + 1) * 4);
        dtv = da + up16(T * 4);
        bar = dtv + up16(T * 4);              // mbarriers: MMA, state rows, x tiles 0 / 1
        tptr = bar + 32;
        total = tptr + 16 + 1024;             // slack for aligning the base
    }
};

// Per-(row, group) tables of the tensor-core form: parents, path checks, C in the
// operand layout, path pairs (pj: path node, pi: node) and C_i . B_j of every pair. All
// of the row's loads are issued at once: C rows into the operand layout and B rows into
// the piece buffer (free between items; 16-byte chunks XOR-swizzled by the row) by
// cp.async, parents and depths into registers; the C . B products then read shared
// memory only. The staged B rows also give the stash its B: the shares of heads hh0 ..
// hh1 (indices within the group) of this CTA's items, each head's share being elements
// [T N hh / hpg, T N (hh + 1) / hpg) of the row's [T][N] block.
//
// Invariant the kernel relies on when it skips an item's closing barrier: before its
// first __syncthreads this function writes only par (plain stores) and, by cp.async, the
// C operand and the piece buffer, which the finished item's MMAs no longer read. It must
// not touch an x tile, cb, pj, cnt, off, sdA or sdt before that barrier, because slower
// threads may still be writing the previous item's outputs out of its x tile.
template <int N>
__device__ void stage_row_tc(const TreeArgs &ta, const TcLayout &lay, uint8_t *sm, int b, int g,
                             bool reporter, int hh0, int hh1)
{
    constexpr int CPR = N / 8;                // 16-byte chunks per bf16 row
    const DecodeArgs &a = ta.d;
    const int T = ta.T, G = a.G, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *cb = reinterpret_cast<float *>(sm + lay.cb);
    uint8_t *pj = sm + lay.pj;
    uint8_t *pi = sm + lay.pi;
    uint8_t *bst = sm + lay.sp;               // B rows of the row's nodes
    int *par = reinterpret_cast<int *>(sm + lay.par);
    int *cnt = reinterpret_cast<int *>(sm + lay.cnt);
    int *off = reinterpret_cast<int *>(sm + lay.off);
    const uint16_t *Cg = static_cast<const uint16_t *>(a.C);
    const uint16_t *Bg = static_cast<const uint16_t *>(a.B);

    for (int k = tid; k < 128 * CPR; k += kTcThreads) {
        const int i = k / CPR, c = k % CPR;
        uint8_t *dst = sm + lay.ca + sw128_off(i, c, 128 * 128);
        if (i < T)
            cp_async16(dst, Cg + (((int64_t)b * T + i) * G + g) * N + c * 8);
        else
            *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
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
    }
    __syncthreads();
    if (tid < T) {
        const int c = cnt[tid], o = off[tid];
        int j = tid;
        for (int k = 0; k < c; ++k) {
            pj[o + k] = static_cast<uint8_t>(j);
            pi[o + k] = static_cast<uint8_t>(tid);
            j = par[j];
        }
    }
    cp_async_wait_all();                      // C and B rows landed
    __syncthreads();
    const int total = off[T];
    for (int p = tid; p < total; p += kTcThreads) {
        const int i = pi[p], j = pj[p];
        const uint8_t *brow = bst + j * (N * 2);
        float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < CPR; ++c) {
            const uint4 cv = *reinterpret_cast<const uint4 *>(sm + lay.ca + sw128_off(i, c, 128 * 128));
            const uint4 bv = *reinterpret_cast<const uint4 *>(brow + ((c ^ (j & 7)) << 4));
            float fc[8], fb[8];
            Vec16<__nv_bfloat16>::unpack(cv, fc);
            Vec16<__nv_bfloat16>::unpack(bv, fb);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                s[e & 3] = fmaf(fc[e], fb[e], s[e & 3]);
        }
        cb[p] = (s[0] + s[1]) + (s[2] + s[3]);
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
        const int o = sw128_off(r, c, kTile * 128);
#pragma unroll
        for (int p = 0; p < NPC; ++p) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * q], f[2 * q + 1]);
                const float2 back = __bfloat1622float2(h);
                f[2 * q] -= back.x;            // exact: the piece is within 2^-8 of f
                f[2 * q + 1] -= back.y;
                memcpy(&w[q], &h, 4);
            }
            *reinterpret_cast<uint4 *>(sm + lay.sp + p * (kTile * N * 2) + o) =
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

// The x tile: one copy per node row (rows 16-byte aligned), spread over nt issuing
// threads (this one is t; t = 0 arms the barrier).
template <typename X>
__device__ __forceinline__ void bulk_x(const TreeArgs &ta, const TcLayout &lay, uint8_t *sm,
                                       const Item &u, int xbuf, uint64_t *bar, int t, int nt,
                                       uint32_t extra)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T;
    constexpr int es = (int)sizeof(X);
    const uint32_t rb = (uint32_t)(u.rows * es);
    if (t == 0)
        mbar_arrive_expect_tx(bar, rb * (uint32_t)T + extra);
    for (int i = t; i < T; i += nt)
        bulk_load(sm + lay.xs + xbuf * lay.xbytes + i * kXS * es,
                  static_cast<const X *>(a.x) + (((int64_t)u.b * T + i) * a.H + u.h) * a.Dm +
                      u.row0,
                  rb, bar);
}

// 16 consecutive x values of node i from dim row d0 of an x tile, and the same positions
// overwritten (rounded to X).
template <typename X>
__device__ __forceinline__ void x_seg16(const uint8_t *xs, int i, int d0, float (&f)[16])
{
    constexpr int per = 16 / (int)sizeof(X);
    const uint4 *p = reinterpret_cast<const uint4 *>(xs + (i * kXS + d0) * (int)sizeof(X));
#pragma unroll
    for (int q = 0; q < 16 / per; ++q)
        Vec16<X>::unpack(p[q], f + per * q);
}

template <typename X>
__device__ __forceinline__ void put_seg16(uint8_t *xs, int i, int d0, const float (&y)[16])
{
    constexpr int per = 16 / (int)sizeof(X);
    uint4 *p = reinterpret_cast<uint4 *>(xs + (i * kXS + d0) * (int)sizeof(X));
#pragma unroll
    for (int q = 0; q < 16 / per; ++q)
        p[q] = Vec16<X>::pack(y + per * q);
}

// U of the item (x widened to fp32): 16 bytes of the tile per task, 16-byte stores; thread
// t of the nt taking part.
template <typename X>
__device__ void stash_u_tc(const TreeArgs &ta, const Item &u, const uint8_t *xs, int t, int nt)
{
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, Dm = a.Dm;
    constexpr int per = 16 / (int)sizeof(X);              // x values per task
    if ((Dm & 3) == 0 && (reinterpret_cast<uintptr_t>(ta.st_U) & 15) == 0) {
        for (int e = t; e < T * (kTile / per); e += nt) {
            const int i = e / (kTile / per), d = per * (e % (kTile / per));
            if (d < u.rows) {
                float f[per];
                Vec16<X>::unpack(*reinterpret_cast<const uint4 *>(xs + (i * kXS + d) * (int)sizeof(X)), f);
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
                    xs_at(xs, a.x_dtype, i * kXS + d);
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

// ocopy: out rows are 16-byte aligned, so the outputs go out through the x tile as whole
// rows (each node's dim rows are contiguous in out); otherwise each thread stores its own.
template <typename S, typename X, int N>
__global__ void __launch_bounds__(kTcThreads, 1)
ssu_ddtree_tc_kernel(const __grid_constant__ TreeArgs ta, const int dtiles, const int64_t nitems,
                     const int nxb, const int xasync, const int ocopy)
{
    constexpr int NPC = Pieces<S>::n;
    constexpr int es_x = (int)sizeof(X);
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, kTile);
    extern __shared__ __align__(16) uint8_t sm_dyn[];
    uint8_t *sm = sm_dyn + ((1024 - (smem_u32(sm_dyn) & 1023)) & 1023);
    const DecodeArgs &a = ta.d;
    const int T = ta.T, H = a.H, Dm = a.Dm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const TcLayout lay(T, N, es_x, (int)sizeof(S), NPC, nxb);
    const float *cb = reinterpret_cast<const float *>(sm + lay.cb);
    const uint8_t *pj = sm + lay.pj;
    const int *cnt = reinterpret_cast<const int *>(sm + lay.cnt);
    const int *off = reinterpret_cast<const int *>(sm + lay.off);
    float *sdA = reinterpret_cast<float *>(sm + lay.da);
    float *sdt = reinterpret_cast<float *>(sm + lay.dtv);
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
    // this thread's node (TMEM lane) and its 16 dim rows (TMEM columns)
    const int ni = 32 * (warp & 3) + lane, d0 = 16 * (warp >> 2);
    const uint32_t taddr = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)d0;
    uint32_t phase = 0;                  // parity of the MMA barrier's next phase
    bool mma_out = false;                // an MMA wait gave up (its phase is still awaited)
    // copies in flight (uniform): state rows, x tiles by buffer bit; parities likewise
    uint32_t s_out = 0, x_out = 0, sph = 0, xph = 0;

    const bool x_mid = xasync && nxb == 2;
    int64_t first, last;
    cta_range(nitems, nitems / a.active, a.active, first, last);
    auto xbuf_of = [&](int64_t it) { return nxb == 2 ? (int)((it - first) & 1) : 0; };
    // copies of item w: the state block by thread 0, the x rows one per thread from the
    // top thread down (measured: issuing them from warps 0-3, which also issue the MMAs
    // and hold the shallowest nodes, makes the launch 7 % slower)
    const int xt = kTcThreads - 1 - tid;
    auto issue = [&](const Item &w, int64_t wit, bool with_x) {
        const int xb = xbuf_of(wit);
        bulk_raw<S, N>(ta, lay, sm, w, sbar, tid == 0,
                       fault_tx(kFaultTreeState, -1, (int)(wit - first)));
        if (with_x)
            bulk_x<X>(ta, lay, sm, w, xb, xbar + xb, xt, kTcThreads,
                      fault_tx(kFaultTreeX, -1, (int)(wit - first)));
        s_out = 1;
        if (with_x)
            x_out |= 1u << xb;
    };
    Item u = item_at(ta, first < last ? first : 0, dtiles);
    float dt_next = 0.f;                 // node tid's dt and the head's scalars, next item
    HeadVals hv_next = {0.f, 0.f, 0.f};
    if (first < last && u.valid(a.P)) {
        issue(u, first, xasync);
        dt_next = dt_of(ta, u);
        hv_next = head_vals(a, u.h);
    }
    int cur_b = -1, cur_g = -1;
    Item v = u;
    for (int64_t it = first; it < last; ++it, u = v) {
        const bool has_next = it + 1 < last;
        if (has_next)
            v = item_after(ta, u, dtiles);
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
                issue(v, it + 1, xasync);
                dt_next = dt_of(ta, v);
                hv_next = head_vals(a, v.h);
            }
            continue;
        }
        // (every thread passed the previous item's closing barrier)
        uint8_t *xs = sm + lay.xs + xbuf_of(it) * lay.xbytes;
        if (u.b != cur_b || u.g != cur_g) {
            // heads of (u.b, u.g) whose dim tile 0 lies in this CTA's range: their B stash
            const int hpg = H / a.G;
            const int64_t rs = (int64_t)u.b * H * dtiles;              // the row's item 0
            const int64_t i0 = (first > rs ? first : rs) - rs;
            const int64_t i1 = (last < rs + (int64_t)H * dtiles ? last : rs + (int64_t)H * dtiles) - rs;
            const int hlo = max((int)((i0 + dtiles - 1) / dtiles), u.g * hpg);
            const int hhi = min((int)((i1 - 1) / dtiles), (u.g + 1) * hpg - 1);
            stage_row_tc<N>(ta, lay, sm, u.b, u.g, u.h == 0 && u.dtile == 0, hlo - u.g * hpg,
                            hhi - u.g * hpg);
            cur_b = u.b;
            cur_g = u.g;
        }
        if (!xasync)
            stage_x_plain<kTcThreads>(ta, xs, u);
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
        node_values(ta, sdA, sdt, u, dt_next, hv);
        __syncthreads();
        if (tid == 0 && !fault_tx(kFaultTreeMma, -1, (int)(it - first))) {
            tc_fence_after();
            const uint32_t base = smem_u32(sm);
            uint32_t acc = 0;
#pragma unroll
            for (int p = NPC - 1; p >= 0; --p)        // smallest piece first
#pragma unroll
                for (int kb = 0; kb < N / 64; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = desc_k_sw128(base + lay.ca + kb * 16384 + kk * 32);
                        const uint64_t bd = desc_k_sw128(base + lay.sp + p * (kTile * N * 2) +
                                                         kb * (kTile * 128) + kk * 32);
                        tc_mma_bf16(tmem, ad, bd, kIdesc, acc);
                        acc = 1;
                    }
            tc_commit(bar);
        }
        if (next_valid) {                // raw staging consumed by the split
            issue(v, it + 1, x_mid);
            dt_next = dt_of(ta, v);
            hv_next = head_vals(a, v.h);
        }
        stash_u_tc<X>(ta, u, xs, tid, kTcThreads);

        // path sums of node ni over rows d0 .. d0 + 15 while the MMAs run
        float ps[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
            ps[e] = 0.f;
        float wi = 1.f;
        const int cn = ni < T ? cnt[ni] : 0, o = ni < T ? off[ni] : 0;
        for (int k = 0; k < cn; ++k) {
            const int j = pj[o + k];
            const float cf = wi * sdt[j] * cb[o + k];
            wi *= sdA[j];
            float xv[16];
            x_seg16<X>(xs, j, d0, xv);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                ps[e] = fmaf(cf, xv[e], ps[e]);
        }
        const bool ok = mbar_wait(bar, phase);
        if (__syncthreads_or(!ok)) {     // the MMAs never completed: give up on the launch
            if (tid == 0 && a.err)
                atomicOr(a.err, SSU_FLAG_TIMEOUT);
            mma_out = true;
            break;
        }
        phase ^= 1u;
        tc_fence_after();
        float dv[16];
        tmem_ld16(taddr, dv);
        const bool mine = ni < T && d0 < u.rows;
        float y[16];
        if (mine) {
            float xv[16];
            x_seg16<X>(xs, ni, d0, xv);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                y[e] = cn > 0 ? fmaf(wi, dv[e], ps[e]) + hv.D * xv[e] : 0.f;
        }
        tc_fence_before();
        if (ocopy) {
            if (mine)
                put_seg16<X>(xs, ni, d0, y);
            fence_async_smem();          // these writes before any copy refills the tile
            __syncthreads();             // the tile holds every output of the item
            const int cpr = u.rows * es_x / 16;
            X *og = static_cast<X *>(a.out);
            for (int k = tid; k < T * cpr; k += kTcThreads) {
                const int i = k / cpr, c = k % cpr;
                *reinterpret_cast<uint4 *>(og + (((int64_t)u.b * T + i) * H + u.h) * Dm +
                                           u.row0 + c * (16 / es_x)) =
                    *reinterpret_cast<const uint4 *>(xs + i * kXS * es_x + c * 16);
            }
        } else if (mine) {
            const int64_t base = (((int64_t)u.b * T + ni) * H + u.h) * Dm + u.row0 + d0;
#pragma unroll
            for (int e = 0; e < 16; ++e)
                if (d0 + e < u.rows)
                    st_f32(a.out, a.x_dtype, base + e, y[e]);
        }
        // Every read of this item's buffers done. Not needed when the x tile is double-
        // buffered and the next item is valid: until the next item's first barrier a
        // thread writes only buffers the output copy-out does not read (par, and by
        // cp.async the C operand and the piece buffer: the invariant stated at
        // stage_row_tc), and this item's x tile is refilled only after that barrier.
        // The parity cases with several items per CTA crossing a (row, group) change
        // (tests/test_gpu_ddtree.py, many rows over groups and dim tiles) run this path.
        if (!(x_mid && next_valid))
            __syncthreads();
        if (next_valid && xasync && !x_mid) {
            bulk_x<X>(ta, lay, sm, v, 0, xbar, xt, kTcThreads,
                      fault_tx(kFaultTreeX, -1, (int)(it + 1 - first)));
            x_out |= 1u;
        }
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
    cp_async_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        tmem_dealloc(tmem, kTcCols);
}

// The tensor-core form when it applies (bf16 B and C with 16-byte aligned C, dstate 64 or
// 128, layout within the shared-memory limit); -1 otherwise.
template <typename S, typename X, int N>
int launch_tc_x(const TreeArgs &a, cudaStream_t stream, int64_t nitems, int dtiles, int xasync)
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
    const int ocopy = (reinterpret_cast<uintptr_t>(a.d.out) & 15) == 0 &&
                      ((int64_t)a.d.Dm * es_x) % 16 == 0;
    const int64_t grid = nitems < f->sms ? nitems : f->sms;
    return launch_kernel(ssu_ddtree_tc_kernel<S, X, N>, (unsigned)grid, kTcThreads, lay.total,
                         stream, a, dtiles, nitems, nxb, xasync, ocopy);
}

template <typename S, int N>
int launch_tc(const TreeArgs &a, cudaStream_t stream, int64_t nitems, int dtiles, int xasync)
{
    if constexpr (N != 64 && N != 128) {
        return -1;
    } else {
        if (a.d.bc_dtype != SSU_BF16 || (reinterpret_cast<uintptr_t>(a.d.C) & 15) != 0)
            return -1;
        switch (a.d.x_dtype) {
        case SSU_F32: return launch_tc_x<S, float, N>(a, stream, nitems, dtiles, xasync);
        case SSU_F16: return launch_tc_x<S, __half, N>(a, stream, nitems, dtiles, xasync);
        default: return launch_tc_x<S, __nv_bfloat16, N>(a, stream, nitems, dtiles, xasync);
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
    const int tc = launch_tc<S, N>(a, stream, nitems, dtiles, xasync);
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
