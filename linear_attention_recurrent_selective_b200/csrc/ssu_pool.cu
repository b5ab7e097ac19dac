// ssu_pool.cu -- slot maintenance on a state pool: zero a slot range, copy a slot.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API), invokeMambaStateClear (one
// slot, or every slot when slot is -1), and Recurrent State Manager page, clearSlot /
// clear / copySlotFrom (copy one slot between pools of the same per-slot geometry).
// Both are plain byte streams: 16-byte accesses when both ends are 16-byte aligned,
// a grid of a few CTAs per SM striding over the range.
#include "ssu_common.cuh"

namespace ssu {
namespace {

constexpr int kPoolThreads = 256;

__global__ void __launch_bounds__(kPoolThreads)
clear_kernel(uint8_t *p, int64_t bytes)
{
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    if ((reinterpret_cast<uintptr_t>(p) & 15) == 0) {
        const int64_t nvec = bytes >> 4;
        uint4 *q = reinterpret_cast<uint4 *>(p);
        for (int64_t i = tid; i < nvec; i += stride)
            q[i] = make_uint4(0, 0, 0, 0);
        for (int64_t i = (nvec << 4) + tid; i < bytes; i += stride)
            p[i] = 0;
    } else {
        for (int64_t i = tid; i < bytes; i += stride)
            p[i] = 0;
    }
}

__global__ void __launch_bounds__(kPoolThreads)
copy_kernel(uint8_t *dst, const uint8_t *src, int64_t bytes)
{
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    if (((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15) == 0) {
        const int64_t nvec = bytes >> 4;
        uint4 *d = reinterpret_cast<uint4 *>(dst);
        const uint4 *s = reinterpret_cast<const uint4 *>(src);
        for (int64_t i = tid; i < nvec; i += stride)
            d[i] = s[i];
        for (int64_t i = (nvec << 4) + tid; i < bytes; i += stride)
            dst[i] = src[i];
    } else {
        for (int64_t i = tid; i < bytes; i += stride)
            dst[i] = src[i];
    }
}

unsigned grid_for(int64_t bytes)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (bytes / 16 + kPoolThreads - 1) / kPoolThreads;
    const int64_t cap = (int64_t)sms * 8;
    return (unsigned)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

int launch_clear(void *pool, int64_t bytes, cudaStream_t s)
{
    if (bytes <= 0)
        return SSU_OK;
    clear_kernel<<<grid_for(bytes), kPoolThreads, 0, s>>>(static_cast<uint8_t *>(pool), bytes);
    return SSU_OK;
}

int launch_copy(void *dst, const void *src, int64_t bytes, cudaStream_t s)
{
    if (bytes <= 0 || dst == src)
        return SSU_OK;
    copy_kernel<<<grid_for(bytes), kPoolThreads, 0, s>>>(static_cast<uint8_t *>(dst),
                                                          static_cast<const uint8_t *>(src),
                                                          bytes);
    return SSU_OK;
}

}  // namespace ssu
