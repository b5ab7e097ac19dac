// ssu_common.cuh -- shared device helpers and launch descriptors for libssu (sm_100a).
//
// Storage types follow the Selective State Update page of the TensorRT-Edge-LLM C++ API:
// the state pool is half or float, A/dt/D/dt_bias are fp32, and x/B/C/z/out may be fp32,
// fp16 or bf16. Every value is widened to fp32 for arithmetic and rounded to nearest
// even once when stored.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>

#include "ssu.h"

namespace ssu {

// ---------------------------------------------------------------- launching

constexpr int kMaxDevices = 64;

// The calling thread's current device, or -1 when it cannot be had or lies beyond the
// per-device caches below.
inline int current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return -1;
    return dev;
}

// Launch `kernel` on `stream` and return the status of this launch alone: an error left
// behind by unrelated earlier work in the calling thread is neither reported here nor
// cleared.
template <typename... KArgs, typename... Args>
int launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                  cudaStream_t stream, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess
               ? SSU_OK
               : SSU_ERR_CUDA;
}

// The same, as a programmatic dependent launch: the kernel may start while the previous
// kernel on the stream still runs (once that kernel's CTAs have all signalled
// griddepcontrol.launch_dependents, or exited), and must execute griddepcontrol.wait
// before it touches anything the previous kernel writes or still reads.
template <typename... KArgs, typename... Args>
int launch_kernel_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t stream, Args &&...args)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess
               ? SSU_OK
               : SSU_ERR_CUDA;
}

// griddepcontrol: let the dependent kernel launch (primary side), and wait until every
// prerequisite kernel has completed and its memory is visible (dependent side; returns at
// once for a kernel launched without a programmatic dependency).
__device__ __forceinline__ void grid_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// What a launch needs to know about the device, found once per process, kernel and
// device under std::call_once (so concurrent first calls from several host threads are
// safe): the SM count, the kernel's dynamic shared-memory limit raised to `smem` bytes,
// and how many CTAs of `threads` threads with `smem` bytes fit on one SM. This cache of
// device facts is the only host state the library keeps; it never affects results.
struct KernelFacts {
    int sms = 0;
    int blocks_per_sm = 0;
    int status = SSU_ERR_CUDA;
};

template <auto kernel>
const KernelFacts *kernel_facts(int threads, int smem)
{
    static std::once_flag once[kMaxDevices];
    static KernelFacts facts[kMaxDevices];
    const int dev = current_device();
    if (dev < 0)
        return nullptr;
    std::call_once(once[dev], [&] {
        KernelFacts f;
        int n = 0, occ = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) ==
                cudaSuccess &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem) ==
                cudaSuccess &&
            n > 0 && occ > 0) {
            f.sms = n;
            f.blocks_per_sm = occ;
            f.status = SSU_OK;
        }
        facts[dev] = f;
    });
    return &facts[dev];
}

#ifdef SSU_WAIT_TEST
// Test build only (libssu_waittest.so): which bounded wait is made to run out, and the
// limit of every wait. site 0 injects nothing; warp < 0 matches every warp of the CTA;
// index counts the wait's instances within that CTA (or warp).
struct WaitFault {
    unsigned long long limit_ns;
    int site, block, warp, index;
};
// one per translation unit that holds bounded waits
int wait_fault_set_decode(const WaitFault &f);
int wait_fault_set_replay(const WaitFault &f);
int wait_fault_set_conv(const WaitFault &f);
int wait_fault_set_gdn(const WaitFault &f);
int wait_fault_set_prefill(const WaitFault &f);
int wait_fault_set_prefill_tc(const WaitFault &f);
int wait_fault_set_ddtree(const WaitFault &f);
#endif

// ---------------------------------------------------------------- launch descriptors

struct DecodeArgs {
    const void *x;
    const float *A;
    const void *B;
    const void *C;
    const float *dt;
    const float *dt_bias;
    const float *D;
    const void *z;
    void *state;
    void *out;
    const int32_t *idx;
    int32_t *err;
    int64_t slot_stride;
    int32_t P, batch, active, H, G, Dm, N;
    int x_dtype, bc_dtype, softplus;
};

struct PrefillArgs {
    DecodeArgs d;             // x/B/C/dt/z/out carry a token axis [batch, T, ...]
    const int32_t *ctx;       // contextLengths [batch] or NULL
    float *st_dA, *st_U, *st_B, *st_dt;  // replay stash, all or none
    int32_t T;
};

struct ReplayArgs {
    const ssu_replay_layer *layers;   // device array [num_layers], or NULL: one layer below
    int32_t num_layers;
    void *state;
    const float *st_dA, *st_U, *st_B, *st_dt;
    const int32_t *acc;
    const int32_t *idx;
    const int32_t *nodes;     // acceptedNodeIds [batch, max_accept] or NULL (token t = t)
    int32_t *err;
    int64_t slot_stride;
    int32_t P, batch, active, T, H, G, Dm, N, max_accept;
};

struct ConvArgs {
    DecodeArgs d;             // x, B, C unused: the conv outputs take their place
    const void *xbc;          // [batch, conv_dim] raw channels (x, B, C order), x dtype
    const void *w;            // [conv_dim, width], x dtype
    const void *bias;         // [conv_dim] or NULL, x dtype
    void *cstate;             // conv pool, element (s, c, k) at s*cslot + c*cc + k*ck
    int64_t cslot, cc, ck;
    int32_t width, silu;
};

struct GdnArgs {
    const void *q, *k;        // [batch, HK, K], x dtype
    const void *v;            // [batch, HV, V], x dtype
    const void *a, *b;        // decay and beta inputs [batch, HV], x dtype
    const float *A_log;       // [HV]
    const float *dt_bias;     // [HV] or NULL
    float *state;             // fp32 pool [P, HV, V, K]
    void *out;                // [batch, HV, V], x dtype
    const int32_t *idx;
    int32_t *err;
    int64_t slot_stride;
    float scale;
    int32_t P, batch, active, HK, HV, K, V, x_dtype, l2norm;
};

struct TreeArgs {
    DecodeArgs d;             // x/B/C/dt/out carry a node axis [batch, T, ...]; z unused
    const int32_t *parents;   // treeParentIds [batch, T]
    const int32_t *depths;    // treeDepths [batch, T]
    float *st_dA, *st_U, *st_B, *st_dt;
    int32_t T;
};

// Host launchers, one per kernel family; each returns SSU_OK or SSU_ERR_UNSUPPORTED.
int launch_decode(const DecodeArgs &a, int state_dtype, cudaStream_t s);
int launch_prefill(const PrefillArgs &a, int state_dtype, cudaStream_t s);
int launch_prefill_tc(const PrefillArgs &a, int state_dtype, cudaStream_t s);  // -1: n/a
int launch_replay(const ReplayArgs &a, int state_dtype, cudaStream_t s);
int launch_ddtree(const TreeArgs &a, int state_dtype, cudaStream_t s);
int launch_conv_decode(const ConvArgs &a, int state_dtype, cudaStream_t s);
int launch_gdn_decode(const GdnArgs &a, cudaStream_t s);
int launch_clear(void *pool, int64_t bytes, cudaStream_t s);
int launch_copy(void *dst, const void *src, int64_t bytes, cudaStream_t s);
int launch_clear_layers(const ssu_layer_states *layers, int32_t num_layers, int32_t P,
                        int32_t slot, int64_t rec_bytes, int64_t conv_bytes, cudaStream_t s);
int launch_gather(const void *pool, int64_t slot_bytes, int32_t P, void *dense,
                  const int32_t *idx, int32_t active, int scatter, int32_t *err,
                  cudaStream_t s);
int launch_check_indices(const int32_t *idx, int32_t active, int32_t P, int32_t *err,
                         cudaStream_t s);

// ---------------------------------------------------------------- scalar access

__device__ __forceinline__ float ld_f32(const void *p, int dtype, int64_t i)
{
    if (dtype == SSU_BF16)
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
    if (dtype == SSU_F16)
        return __half2float(static_cast<const __half *>(p)[i]);
    return static_cast<const float *>(p)[i];
}

__device__ __forceinline__ void st_f32(void *p, int dtype, int64_t i, float v)
{
    if (dtype == SSU_BF16)
        static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
    else if (dtype == SSU_F16)
        static_cast<__half *>(p)[i] = __float2half_rn(v);
    else
        static_cast<float *>(p)[i] = v;
}

// Raw bits of element i (16-bit types zero-extended), for prefetches whose widening is
// deferred until the value is used, so that no instruction waits on the load early.
__device__ __forceinline__ uint32_t ld_bits(const void *p, int dtype, int64_t i)
{
    if (dtype == SSU_F32)
        return static_cast<const uint32_t *>(p)[i];
    return static_cast<const uint16_t *>(p)[i];
}

__device__ __forceinline__ float bits_f32(uint32_t v, int dtype)
{
    if (dtype == SSU_F32)
        return __uint_as_float(v);
    if (dtype == SSU_BF16)
        return __uint_as_float(v << 16);
    return __half2float(__ushort_as_half(static_cast<unsigned short>(v)));
}

// softplus(v) = log(1 + e^v); above 20 the correction log1p(e^-v) < 2.1e-9 is dropped.
__device__ __forceinline__ float softplus_f(float v)
{
    return v > 20.f ? v : log1pf(expf(v));
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + expf(-z)); }

// dt after the optional bias and the optional softplus (one value per row, token, head)
__device__ __forceinline__ float effective_dt(float dt, const float *bias, int h, int sp)
{
    float v = dt + (bias ? bias[h] : 0.f);
    return sp ? softplus_f(v) : v;
}

// ---------------------------------------------------------------- prefill scheduling

constexpr int kRankMax = 32;    // prefill batches up to this size run longest rows first

// Length used for scheduling a prefill row: padding and out-of-range rows do (almost) no
// work.
__device__ __forceinline__ int prefill_sched_len(const PrefillArgs &pa, int b)
{
    const int slot = pa.d.idx ? pa.d.idx[b] : b;
    if (slot < 0 || slot >= pa.d.P)
        return 0;
    const int L = pa.ctx ? pa.ctx[b] : pa.T;
    return L < 0 ? 0 : (L > pa.T ? pa.T : L);
}

// The row a prefill CTA of rank `rank` takes: with at most kRankMax active rows, rows are
// ranked by decreasing length from the device lengths (ties by index) so that the longest
// scans start first; otherwise row `rank`. Every thread of the CTA calls it (s_len
// [kRankMax] and s_row in shared memory).
__device__ __forceinline__ int prefill_ranked_row(const PrefillArgs &pa, int rank, int *s_len,
                                                  int *s_row)
{
    const int tid = threadIdx.x, active = pa.d.active;
    if (active > kRankMax)
        return rank;
    if (tid < active)
        s_len[tid] = prefill_sched_len(pa, tid);
    __syncthreads();
    if (tid < active) {
        const int mine = s_len[tid];
        int r = 0;
        for (int o = 0; o < active; ++o)
            r += (s_len[o] > mine) || (s_len[o] == mine && o < tid);
        if (r == rank)
            *s_row = tid;
    }
    __syncthreads();
    return *s_row;
}

// ---------------------------------------------------------------- 16-byte state vectors

template <typename S> struct Vec16;

template <> struct Vec16<float> {
    static constexpr int kElems = 4;
    static __device__ __forceinline__ void unpack(const uint4 &v, float *f)
    {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
    static __device__ __forceinline__ uint4 pack(const float *f)
    {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                          __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

template <typename H2, typename Cvt> struct Vec16Half {
    static constexpr int kElems = 8;
    static __device__ __forceinline__ void unpack(const uint4 &v, float *f)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            H2 h;
            memcpy(&h, &w[i], 4);
            float2 p = Cvt::to_f2(h);
            f[2 * i] = p.x;
            f[2 * i + 1] = p.y;
        }
    }
    static __device__ __forceinline__ uint4 pack(const float *f)
    {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            H2 h = Cvt::from_f2(f[2 * i], f[2 * i + 1]);
            memcpy(&w[i], &h, 4);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

struct CvtHalf {
    static __device__ __forceinline__ float2 to_f2(__half2 h) { return __half22float2(h); }
    static __device__ __forceinline__ __half2 from_f2(float a, float b)
    {
        return __floats2half2_rn(a, b);
    }
};
struct CvtBf16 {
    static __device__ __forceinline__ float2 to_f2(__nv_bfloat162 h)
    {
        return __bfloat1622float2(h);
    }
    static __device__ __forceinline__ __nv_bfloat162 from_f2(float a, float b)
    {
        return __floats2bfloat162_rn(a, b);
    }
};

template <> struct Vec16<__half> : Vec16Half<__half2, CvtHalf> {};
template <> struct Vec16<__nv_bfloat16> : Vec16Half<__nv_bfloat162, CvtBf16> {};

// Four consecutive state elements as floats (8- or 16-byte access).
template <typename S> struct Quad;
template <> struct Quad<float> {
    static __device__ __forceinline__ float4 load(const float *p)
    {
        return *reinterpret_cast<const float4 *>(p);
    }
    static __device__ __forceinline__ void store(float *p, float4 v)
    {
        *reinterpret_cast<float4 *>(p) = v;
    }
};
template <typename S, typename H2, typename Cvt> struct QuadHalf {
    static __device__ __forceinline__ float4 load(const S *p)
    {
        uint2 w = *reinterpret_cast<const uint2 *>(p);
        H2 a, b;
        memcpy(&a, &w.x, 4);
        memcpy(&b, &w.y, 4);
        float2 fa = Cvt::to_f2(a), fb = Cvt::to_f2(b);
        return make_float4(fa.x, fa.y, fb.x, fb.y);
    }
    static __device__ __forceinline__ void store(S *p, float4 v)
    {
        H2 a = Cvt::from_f2(v.x, v.y), b = Cvt::from_f2(v.z, v.w);
        uint2 w;
        memcpy(&w.x, &a, 4);
        memcpy(&w.y, &b, 4);
        *reinterpret_cast<uint2 *>(p) = w;
    }
};
template <> struct Quad<__half> : QuadHalf<__half, __half2, CvtHalf> {};
template <> struct Quad<__nv_bfloat16> : QuadHalf<__nv_bfloat16, __nv_bfloat162, CvtBf16> {};

}  // namespace ssu
