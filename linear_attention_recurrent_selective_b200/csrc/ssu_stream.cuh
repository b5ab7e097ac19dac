// ssu_stream.cuh -- the per-warp streaming pipeline shared by the HBM-bound kernels
// (decode and replay), which read every touched state row once and write it once.
//
// Work is cut into "units": up to kUnitRows rows (and at most UT tiles) of one head of
// one batch row's slot. Persistent CTAs of kWarps warps each run an independent pipeline:
// warp w of the grid takes units w, w + W, w + 2W, ... (W = warps in the grid), so all
// warps sweep the pool together in address order. A unit is cut into tiles of up to
// kTileBytes of contiguous state; every warp owns a ring of kStages shared-memory tile
// buffers that the bulk-copy engine fills (cp.async.bulk, completion counted on a
// per-buffer mbarrier), so kStages-1 tiles are in flight while the warp computes on one.
// Lane 0 is the producer: it resolves the pool, slot and any per-row extra (such as an
// accepted length) of the unit after the one it is copying one unit early, so the index
// loads never stall the ring. Multi-layer launches number units layer-major. Rows that touch no state (padding, out-of-range
// index, nothing accepted) complete their buffer's barrier without a copy, which keeps
// the consumer's phase bookkeeping uniform.
#pragma once

#include "ssu_async.cuh"
#include "ssu_common.cuh"

namespace ssu {
namespace stream {

// Pipeline shape; the defaults are the measured best on B200 for the batch-256 decode
// and can be overridden at build time for tuning sweeps.
#ifndef SSU_STREAM_WARPS
#define SSU_STREAM_WARPS 8
#endif
#ifndef SSU_STREAM_STAGES
#define SSU_STREAM_STAGES 3
#endif
constexpr int kWarps = SSU_STREAM_WARPS;    // warps per CTA, each an independent pipeline
constexpr int kStages = SSU_STREAM_STAGES;  // tile buffers per warp
constexpr int kTileBytes = 4096;            // one tile: 8 warp-wide 512-byte accesses
constexpr int kUnitRows = 128;              // at most this many rows per unit

// Geometry of a unit of at most UT tiles (UT * 4 KB of state) for state type S, dstate N.
template <typename S, int N, int UT> struct Geo {
    static constexpr int VEC = Vec16<S>::kElems;                 // elements per 16 bytes
    static constexpr int LPR = (N / VEC) < 32 ? (N / VEC) : 32;  // lanes per state row
    static constexpr int E = N / LPR;                           // elements per lane and row
    static constexpr int NV = E / VEC;                          // 16-byte vectors per lane/row
    static constexpr int RPW = 32 / LPR;                        // rows per warp access
    static constexpr int ELEM = (int)sizeof(S);
    static constexpr int ROW_BYTES = N * ELEM;
    static constexpr int RT = kTileBytes / ROW_BYTES;           // rows per full tile
    static constexpr int RPT = RT / RPW;                        // row accesses per lane/tile
    static constexpr int CR = (UT * RT) < kUnitRows ? (UT * RT) : kUnitRows;
    static constexpr int XR = (CR + 31) / 32;                   // unit rows per lane
    static_assert(RT >= 1 && RPT >= 1 && RPT * RPW == RT, "tile geometry");
    // state column n of vector v, element e for lane-in-row ln
    static __device__ __forceinline__ int col(int v, int ln, int e) { return (v * LPR + ln) * VEC + e; }
};

struct Ring {
    uint64_t full[kStages];
    int slot[kStages];    // slot of the unit whose tile sits in each buffer
    int extra[kStages];   // per-row extra of that unit (e.g. the accepted length)
    int moves[kStages];   // whether that tile was copied
};
static_assert(sizeof(Ring) <= 128, "per-warp control block");

constexpr int kRingBytes = kStages * kTileBytes;
constexpr int kStageBytes = 2 * kUnitRows * 4;           // two per-unit float rows
constexpr int kPerWarpBytes = kRingBytes + kStageBytes + 128;   // a multiple of 128
constexpr int kSmemBytes = kWarps * kPerWarpBytes;

struct Unit {
    int b, h, row0, rows;
};

__device__ __forceinline__ Unit unit_at(int u, int cph, int CR, int H, int Dm)
{
    Unit un;
    const int c = u % cph;
    const int v = u / cph;
    un.h = v % H;
    un.b = v / H;
    un.row0 = c * CR;
    un.rows = min(CR, Dm - un.row0);
    return un;
}

// A unit of a multi-layer launch: units are numbered layer-major, upl units per layer.
struct LUnit {
    Unit un;
    int layer;
};

__device__ __forceinline__ LUnit lunit_at(int u, int upl, int cph, int CR, int H, int Dm)
{
    LUnit lu;
    lu.layer = u / upl;
    lu.un = unit_at(u - lu.layer * upl, cph, CR, H, Dm);
    return lu;
}

// Units numbered in order: layer-major, then row, head and dim chunk.
struct UnitsInOrder {
    __device__ __forceinline__ LUnit unit(int u, int upl, int cph, int CR, int H, int Dm) const
    {
        return lunit_at(u, upl, cph, CR, H, Dm);
    }
};

// What the producer needs to know about a unit: the base of its layer's pool, its slot and
// a per-row extra (such as an accepted length).
struct UnitRes {
    const char *pool;
    int slot;
    int extra;
};

// Per-warp views of the dynamic shared memory.
struct WarpViews {
    uint8_t *ring;     // kStages tile buffers
    float *f0, *f1;    // two [kUnitRows] float rows for per-unit staging
    Ring *ctl;
};

__device__ __forceinline__ WarpViews warp_views(uint8_t *smem, int warp)
{
    WarpViews w;
    w.ring = smem + warp * kPerWarpBytes;
    w.f0 = reinterpret_cast<float *>(w.ring + kRingBytes);
    w.f1 = w.f0 + kUnitRows;
    w.ctl = reinterpret_cast<Ring *>(w.f1 + kUnitRows);
    return w;
}

// Lane 0's side of a warp's pipeline. `Rows` numbers the units, maps a unit to its pool,
// slot and extra, and says whether the unit moves state:
//   LUnit unit(int u, int upl, int cph, int CR, int H, int Dm) const;
//   UnitRes resolve(const LUnit &lu) const;  bool moves(const UnitRes &r) const;
template <typename G, int N, typename Rows> struct Producer {
    int k;        // position in this warp's unit sequence
    int j;        // next tile within the unit
    int tiles;    // tiles of the current unit
    UnitRes cur;  // the current unit
    UnitRes nxt;  // the next unit (resolved one unit early)
    int issued;   // tiles issued so far

    __device__ void start(const Rows &rows, int gw, int nw, int upl, int cph, int nunits, int H,
                          int Dm)
    {
        k = 0;
        j = 0;
        issued = 0;
        tiles = 0;
        cur = UnitRes{nullptr, -1, 0};
        nxt = UnitRes{nullptr, -1, 0};
        if (gw < nunits) {
            const LUnit lu = rows.unit(gw, upl, cph, G::CR, H, Dm);
            cur = rows.resolve(lu);
            tiles = (lu.un.rows + G::RT - 1) / G::RT;
            if (gw + nw < nunits)
                nxt = rows.resolve(rows.unit(gw + nw, upl, cph, G::CR, H, Dm));
        }
    }

    __device__ void issue(const Rows &rows, int64_t slot_stride, int gw, int nw, int upl, int cph,
                          int nunits, int H, int Dm, const WarpViews &w, int s)
    {
        const int u = gw + k * nw;
        if (u >= nunits)
            return;
        const Unit un = rows.unit(u, upl, cph, G::CR, H, Dm).un;
        w.ctl->slot[s] = cur.slot;
        w.ctl->extra[s] = cur.extra;
        w.ctl->moves[s] = rows.moves(cur);
        const uint32_t extra = fault_tx(kFaultStream, (int)(threadIdx.x >> 5), issued);
        if (w.ctl->moves[s]) {
            const int nr = min(G::RT, un.rows - j * G::RT);
            const uint32_t bytes = (uint32_t)(nr * G::ROW_BYTES);
            const char *src = cur.pool + ((int64_t)cur.slot * slot_stride +
                                          ((int64_t)un.h * Dm + un.row0 + j * G::RT) * N) *
                                             G::ELEM;
            mbar_arrive_expect_tx(&w.ctl->full[s], bytes + extra);
            bulk_load(w.ring + s * kTileBytes, src, bytes, &w.ctl->full[s]);
        } else if (extra) {
            mbar_arrive_expect_tx(&w.ctl->full[s], extra);
        } else {
            mbar_arrive(&w.ctl->full[s]);
        }
        ++issued;
        if (++j == tiles) {                  // move to this warp's next unit
            j = 0;
            ++k;
            const int u2 = gw + k * nw;
            if (u2 < nunits) {
                cur = nxt;
                tiles = (rows.unit(u2, upl, cph, G::CR, H, Dm).un.rows + G::RT - 1) / G::RT;
                if (u2 + nw < nunits)
                    nxt = rows.resolve(rows.unit(u2 + nw, upl, cph, G::CR, H, Dm));
            }
        }
    }
};

// Row sums of a tile. v[i] holds this lane's partial sum of its i-th row (RPT rows, each
// spread over the LPR lanes ln = 0..LPR-1 of a row group). With RPT <= LPR the sums are
// reduced by a transposing butterfly: at each of the first log2(RPT) steps a lane keeps
// half of its values and sends the other half to its partner (RPT - 1 shuffles in all),
// then plain butterfly steps finish the sum; otherwise every row takes its own butterfly.
// Returns the full sum of row `row` of this lane; `writer` marks one lane per row.
template <int RPT, int LPR>
__device__ __forceinline__ float row_sums(float (&v)[RPT], int ln, int &row, bool &writer)
{
    if constexpr (RPT <= LPR && RPT > 1) {
        int base = 0;
#pragma unroll
        for (int c = RPT, o = LPR / 2; c > 1; c >>= 1, o >>= 1) {
            const bool hi = (ln & o) != 0;
            const int half = c / 2;
#pragma unroll
            for (int k = 0; k < half; ++k) {
                const float keep = hi ? v[k + half] : v[k];
                const float send = hi ? v[k] : v[k + half];
                v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
            base += hi ? half : 0;
        }
        float t = v[0];
#pragma unroll
        for (int o = LPR / RPT / 2; o > 0; o >>= 1)
            t += __shfl_xor_sync(0xffffffffu, t, o);
        row = base;
        writer = (ln & (LPR / RPT - 1)) == 0;
        return t;
    } else {
        // one butterfly per row; the caller asks for each row in turn through `row`
        float t = v[row];
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1)
            t += __shfl_xor_sync(0xffffffffu, t, o);
        writer = ln == 0;
        return t;
    }
}

// Initialise the warp's ring barriers (lane 0) and make them visible to the copy engine.
__device__ __forceinline__ void init_ring(const WarpViews &w, int lane)
{
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kStages; ++s)
            mbar_init(&w.ctl->full[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
}

// Wait for consumed-tile number c; on a (never expected) timeout, report it, wait (each
// wait bounded again) for every tile this warp still has in flight, so that no copy
// outlives the warp unless its barrier also gives up, and return false. The verdict is
// warp-uniform.
__device__ __forceinline__ bool wait_tile(const WarpViews &w, int c, int issued_lane0,
                                          int lane, int32_t *err)
{
    const int s = c % kStages;
    if (__all_sync(0xffffffffu, mbar_wait(&w.ctl->full[s], (uint32_t)(c / kStages) & 1u)))
        return true;
    if (lane == 0 && err)
        atomicOr(err, SSU_FLAG_TIMEOUT);
    const int issued = __shfl_sync(0xffffffffu, issued_lane0, 0);
    for (int cc = c; cc < issued; ++cc)
        mbar_wait(&w.ctl->full[cc % kStages], (uint32_t)(cc / kStages) & 1u);
    return false;
}

// Grid size for a persistent launch: as many CTAs as fit, no more than the work needs;
// -1 when the device could not be queried (the launcher then reports SSU_ERR_CUDA).
template <auto kernel>
int persistent_grid(int64_t nunits)
{
    const KernelFacts *f = kernel_facts<kernel>(kWarps * 32, kSmemBytes);
    if (!f || f->status != SSU_OK)
        return -1;
    const int64_t want = (nunits + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)f->sms * f->blocks_per_sm;
    return (int)(want < cap ? want : cap);
}

}  // namespace stream
}  // namespace ssu
