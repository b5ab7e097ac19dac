// ssu_gdn.cu -- gated delta-rule decode over a paged fp32 state pool (the recurrent core
// of the FlashInfer page flashinfer.gdn_fused_decode_step).
//
// Per active row b and value head hv (key head hk = hv / (HV / HK)), with the key head's
// q and k L2-normalised (sum of squares + 1e-6) and q scaled (default 1/sqrt(K)):
//     alpha = exp(-exp(A_log[hv]) * softplus(a[b,hv] + dt_bias[hv])),  beta = sigmoid(b[b,hv])
//     for every state row i (V rows of K columns, K innermost):
//         u = alpha * (S_i . k);  d = beta * (v_i - u)
//         S_i <- alpha * S_i + d * k;   out_i = S_i . q = alpha * (S_i . q) + d * (k . q)
// The page's padding contract holds: a negative state index touches no state and writes
// zeros, an index >= P is skipped and reported (SSU_FLAG_INDEX_RANGE).
//
// Like the Mamba decode, the step reads and writes every state element once and is bound
// by HBM, so it runs on the per-warp bulk-copy pipeline of ssu_stream.cuh: units of up to
// 64 rows of one value head, tiles of 4 KB streamed through a ring of shared-memory
// buffers. Per unit the lane's columns of q and k are normalised with warp shuffles (every
// lane group holds the same columns), k . q and the gates are formed once; per tile the
// dot products S_i . k and S_i . q of all rows come from one pass over the rows in
// registers and one transposing butterfly each (ssu_stream.cuh, row_sums), the row's
// owner lane forms d, every lane fetches d of its rows, and the updated rows are written
// straight back.
#include "ssu_stream.cuh"

namespace ssu {
namespace {

using namespace stream;

constexpr int kUT = 8;

struct GdnRows : UnitsInOrder {
    const void *pool;
    const int32_t *idx;
    int32_t P;
    __device__ __forceinline__ UnitRes resolve(const LUnit &lu) const
    {
        return UnitRes{static_cast<const char *>(pool), idx ? idx[lu.un.b] : lu.un.b, 0};
    }
    __device__ __forceinline__ bool moves(const UnitRes &r) const
    {
        return r.slot >= 0 && r.slot < P;
    }
};

// Sum over the LPR lanes that share a row (butterfly; every lane gets the total).
template <int LPR>
__device__ __forceinline__ float group_sum(float v)
{
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

template <int K>
__global__ void __launch_bounds__(kWarps * 32)
gdn_decode_kernel(const __grid_constant__ GdnArgs a, const int cph, const int nunits)
{
    using G = Geo<float, K, kUT>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WarpViews w = warp_views(smem, warp);
    float *vs = w.f0;                           // unit v, [CR]
    float *ys = w.f1;                           // unit outputs, [CR]
    init_ring(w, lane);

    const int H = a.HV, Dm = a.V, vpk = a.HV / a.HK;
    const int gw = blockIdx.x * kWarps + warp;
    const int nw = gridDim.x * kWarps;
    const GdnRows rows{{}, a.state, a.idx, a.P};
    Producer<G, K, GdnRows> prod;
    if (lane == 0) {
        prod.start(rows, gw, nw, nunits, cph, nunits, H, Dm);
#pragma unroll
        for (int s = 0; s < kStages; ++s)
            prod.issue(rows, a.slot_stride, gw, nw, nunits, cph, nunits, H, Dm, w, s);
    }

    const int ln = lane % G::LPR, sub = lane / G::LPR;
    int c = 0;                                  // tiles consumed by this warp
    for (int u = gw; u < nunits; u += nw) {
        const Unit un = unit_at(u, cph, G::CR, H, Dm);
        const int tiles = (un.rows + G::RT - 1) / G::RT;
        const int64_t orow = ((int64_t)un.b * H + un.h) * Dm + un.row0;

        // ---- per-unit inputs: normalised q and k columns of the lane, gates, v rows
        float kn[G::E], qn[G::E];
        {
            const int64_t kb = ((int64_t)un.b * a.HK + un.h / vpk) * K;
            float nk = 0.f, nq = 0.f;
#pragma unroll
            for (int v = 0; v < G::NV; ++v)
#pragma unroll
                for (int e = 0; e < G::VEC; ++e) {
                    const int j = G::col(v, ln, e);
                    kn[v * G::VEC + e] = ld_f32(a.k, a.x_dtype, kb + j);
                    qn[v * G::VEC + e] = ld_f32(a.q, a.x_dtype, kb + j);
                    nk = fmaf(kn[v * G::VEC + e], kn[v * G::VEC + e], nk);
                    nq = fmaf(qn[v * G::VEC + e], qn[v * G::VEC + e], nq);
                }
            float fk = 1.f, fq = a.scale;
            if (a.l2norm) {
                fk = rsqrtf(group_sum<G::LPR>(nk) + 1e-6f);
                fq *= rsqrtf(group_sum<G::LPR>(nq) + 1e-6f);
            }
#pragma unroll
            for (int e = 0; e < G::E; ++e) {
                kn[e] *= fk;
                qn[e] *= fq;
            }
        }
        float kq = 0.f;
#pragma unroll
        for (int e = 0; e < G::E; ++e)
            kq = fmaf(kn[e], qn[e], kq);
        kq = group_sum<G::LPR>(kq);
        const int64_t gi = (int64_t)un.b * H + un.h;
        const float av = ld_f32(a.a, a.x_dtype, gi) + (a.dt_bias ? a.dt_bias[un.h] : 0.f);
        const float alpha = expf(-expf(a.A_log[un.h]) * softplus_f(av));
        const float beta = 1.f / (1.f + expf(-ld_f32(a.b, a.x_dtype, gi)));
#pragma unroll
        for (int m = 0; m < G::XR; ++m) {
            const int r = lane + 32 * m;
            if (r < G::CR)
                vs[r] = r < un.rows ? ld_f32(a.v, a.x_dtype, orow + r) : 0.f;
        }
        __syncwarp();

        int slot = -1;
        for (int j = 0; j < tiles; ++j, ++c) {
            if (!wait_tile(w, c, lane == 0 ? prod.issued : 0, lane, a.err))
                return;
            const int s = c % kStages;
            slot = w.ctl->slot[s];
            if (w.ctl->moves[s]) {
                const int rt = min(G::RT, un.rows - j * G::RT);
                const uint8_t *buf = w.ring + s * kTileBytes;
                float *dst = a.state + (int64_t)slot * a.slot_stride +
                             ((int64_t)un.h * Dm + un.row0 + j * G::RT) * K;
                float f[G::RPT][G::E], pk[G::RPT], pq[G::RPT];
#pragma unroll
                for (int i = 0; i < G::RPT; ++i) {
                    const int r = i * G::RPW + sub;
#pragma unroll
                    for (int v = 0; v < G::NV; ++v) {
                        const uint4 q4 = r < rt ? *reinterpret_cast<const uint4 *>(
                                                      buf + r * G::ROW_BYTES + (v * G::LPR + ln) * 16)
                                                : make_uint4(0, 0, 0, 0);
                        Vec16<float>::unpack(q4, &f[i][v * G::VEC]);
                    }
                    pk[i] = pq[i] = 0.f;
#pragma unroll
                    for (int e = 0; e < G::E; ++e) {
                        pk[i] = fmaf(f[i][e], kn[e], pk[i]);
                        pq[i] = fmaf(f[i][e], qn[e], pq[i]);
                    }
                }
                // per-row d = beta (v - alpha S.k) and out = alpha S.q + d k.q
                float d[G::RPT];
                if constexpr (G::RPT <= G::LPR) {
                    // transposing butterflies leave each lane one row's sums; its owner
                    // forms d, and every lane of the row group fetches d of each row
                    int i = 0, i2 = 0;
                    bool wr = false, wr2 = false;
                    const float tk = row_sums<G::RPT, G::LPR>(pk, ln, i, wr);
                    const float tq = row_sums<G::RPT, G::LPR>(pq, ln, i2, wr2);
                    const int r = i * G::RPW + sub;
                    const float dm = r < rt ? beta * (vs[j * G::RT + r] - alpha * tk) : 0.f;
                    if (wr && r < rt)
                        ys[j * G::RT + r] = fmaf(alpha, tq, dm * kq);
#pragma unroll
                    for (int ii = 0; ii < G::RPT; ++ii)
                        d[ii] = __shfl_sync(0xffffffffu, dm,
                                            sub * G::LPR + ii * (G::LPR / G::RPT));
                } else {
#pragma unroll
                    for (int ii = 0; ii < G::RPT; ++ii) {
                        int i = ii;
                        bool wr = false;
                        const float tk = row_sums<G::RPT, G::LPR>(pk, ln, i, wr);
                        const float tq = row_sums<G::RPT, G::LPR>(pq, ln, i, wr);
                        const int r = ii * G::RPW + sub;
                        d[ii] = r < rt ? beta * (vs[j * G::RT + r] - alpha * tk) : 0.f;
                        if (wr && r < rt)
                            ys[j * G::RT + r] = fmaf(alpha, tq, d[ii] * kq);
                    }
                }
#pragma unroll
                for (int i = 0; i < G::RPT; ++i) {
                    const int r = i * G::RPW + sub;
#pragma unroll
                    for (int e = 0; e < G::E; ++e)
                        f[i][e] = fmaf(alpha, f[i][e], d[i] * kn[e]);
                    if (r < rt) {
#pragma unroll
                        for (int v = 0; v < G::NV; ++v)
                            *reinterpret_cast<uint4 *>(dst + (int64_t)r * K + G::col(v, ln, 0)) =
                                Vec16<float>::pack(&f[i][v * G::VEC]);
                    }
                }
            }
            __syncwarp();                        // every lane is done with buffer s
            if (lane == 0)
                prod.issue(rows, a.slot_stride, gw, nw, nunits, cph, nunits, H, Dm, w, s);
        }

        // ---- the unit's outputs, one coalesced store per 32 rows
        if (slot >= a.P) {
            if (lane == 0 && un.h == 0 && un.row0 == 0 && a.err)
                atomicOr(a.err, SSU_FLAG_INDEX_RANGE);
        } else {
#pragma unroll
            for (int m = 0; m < G::XR; ++m) {
                const int r = lane + 32 * m;
                if (r < un.rows)
                    st_f32(a.out, a.x_dtype, orow + r, slot >= 0 ? ys[r] : 0.f);
            }
        }
        __syncwarp();                            // vs / ys are reused by the next unit
    }
}

template <int K>
int launch_k(const GdnArgs &a, cudaStream_t stream)
{
    using G = Geo<float, K, kUT>;
    const int64_t cph = (a.V + G::CR - 1) / G::CR;
    const int64_t nunits = (int64_t)a.active * a.HV * cph;
    if (nunits == 0)
        return SSU_OK;
    if (nunits > 0x7fffffffLL)
        return SSU_ERR_SHAPE;
    const int grid = persistent_grid<gdn_decode_kernel<K>>(nunits);
    if (grid < 0)
        return SSU_ERR_CUDA;
    return launch_kernel(gdn_decode_kernel<K>, grid, kWarps * 32, kSmemBytes, stream, a,
                         (int)cph, (int)nunits);
}

}  // namespace

#ifdef SSU_WAIT_TEST
SSU_WAIT_FAULT_SETTER(wait_fault_set_gdn)
#endif

int launch_gdn_decode(const GdnArgs &a, cudaStream_t s)
{
    switch (a.K) {
    case 8: return launch_k<8>(a, s);
    case 16: return launch_k<16>(a, s);
    case 32: return launch_k<32>(a, s);
    case 64: return launch_k<64>(a, s);
    case 128: return launch_k<128>(a, s);
    case 256: return launch_k<256>(a, s);
    default: return SSU_ERR_UNSUPPORTED;
    }
}

}  // namespace ssu
