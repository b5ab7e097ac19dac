// ssu_pool.cu -- slot maintenance on a state pool: zero a slot range, copy a slot.
//
// Selective State Update page (TensorRT-Edge-LLM C++ API), invokeMambaStateClear (one
// slot, or every slot when slot is -1), and Recurrent State Manager page, clearSlot /
// clear / copySlotFrom (copy one slot between pools of the same per-slot geometry).
// Plus the multi-layer clear (invokeMambaStateClear over MambaStateLayerInfo arrays) and
// the gather/scatter of active rows (invokeMambaStateGather / Scatter) of the Selective
// State Update page. All are plain byte streams: 16-byte accesses when both ends are
// 16-byte aligned, grid-stride loops.
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

// invokeMambaStateClear: every layer's recurrent (and convolution) slot range is zeroed in
// one launch; blockIdx.y picks the layer and the state kind.
__global__ void __launch_bounds__(kPoolThreads)
clear_layers_kernel(const ssu_layer_states *layers, int32_t slot, int32_t P, int64_t rec_bytes,
                    int64_t conv_bytes)
{
    const int layer = blockIdx.y >> 1, kind = blockIdx.y & 1;
    const ssu_layer_states L = layers[layer];
    uint8_t *base = static_cast<uint8_t *>(kind == 0 ? L.recurrent_state : L.conv_state);
    const int64_t sb = kind == 0 ? rec_bytes : conv_bytes;
    if (!base || sb == 0)
        return;
    uint8_t *p = slot < 0 ? base : base + (int64_t)slot * sb;
    const int64_t bytes = slot < 0 ? sb * P : sb;
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

// invokeMambaStateGather / Scatter: blockIdx.y is the batch row; rows with a negative
// index are padding (gather writes zeros), rows with an index >= P are skipped.
__global__ void __launch_bounds__(kPoolThreads)
gather_kernel(const uint8_t *pool, int64_t slot_bytes, int32_t P, uint8_t *dense,
              const int32_t *idx, int scatter, int32_t *err)
{
    const int b = blockIdx.y;
    const int slot = idx ? idx[b] : b;
    if (slot >= P) {
        if (blockIdx.x == 0 && threadIdx.x == 0 && err)
            atomicOr(err, SSU_FLAG_INDEX_RANGE);
        return;
    }
    if (slot < 0 && scatter)
        return;
    uint8_t *drow = dense + (int64_t)b * slot_bytes;
    uint8_t *prow = const_cast<uint8_t *>(pool) + (int64_t)(slot < 0 ? 0 : slot) * slot_bytes;
    const uint8_t *src = scatter ? drow : prow;
    uint8_t *dst = scatter ? prow : drow;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const bool vec = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0;
    const int64_t nvec = vec ? slot_bytes >> 4 : 0;
    for (int64_t i = tid; i < nvec; i += stride)
        reinterpret_cast<uint4 *>(dst)[i] =
            slot < 0 ? make_uint4(0, 0, 0, 0) : reinterpret_cast<const uint4 *>(src)[i];
    for (int64_t i = (nvec << 4) + tid; i < slot_bytes; i += stride)
        dst[i] = slot < 0 ? 0 : src[i];
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
    return launch_kernel(clear_kernel, grid_for(bytes), kPoolThreads, 0, s,
                         static_cast<uint8_t *>(pool), bytes);
}

int launch_clear_layers(const ssu_layer_states *layers, int32_t num_layers, int32_t P,
                        int32_t slot, int64_t rec_bytes, int64_t conv_bytes, cudaStream_t s)
{
    const int64_t per = slot < 0 ? (rec_bytes > conv_bytes ? rec_bytes : conv_bytes) * P
                                 : (rec_bytes > conv_bytes ? rec_bytes : conv_bytes);
    if (per <= 0)
        return SSU_OK;
    if ((int64_t)num_layers * 2 > 65535)
        return SSU_ERR_SHAPE;
    const int64_t want = (per / 16 + kPoolThreads - 1) / kPoolThreads;
    const unsigned gx = (unsigned)(want < 1 ? 1 : (want < 64 ? want : 64));
    return launch_kernel(clear_layers_kernel, dim3(gx, 2 * num_layers), kPoolThreads, 0, s,
                         layers, slot, P, rec_bytes, conv_bytes);
}

int launch_gather(const void *pool, int64_t slot_bytes, int32_t P, void *dense,
                  const int32_t *idx, int32_t active, int scatter, int32_t *err, cudaStream_t s)
{
    if (active > 65535)
        return SSU_ERR_SHAPE;
    const int64_t want = (slot_bytes / 16 + kPoolThreads - 1) / kPoolThreads;
    const unsigned gx = (unsigned)(want < 1 ? 1 : (want < 32 ? want : 32));
    return launch_kernel(gather_kernel, dim3(gx, active), kPoolThreads, 0, s,
                         static_cast<const uint8_t *>(pool), slot_bytes, P,
                         static_cast<uint8_t *>(dense), idx, scatter, err);
}

int launch_copy(void *dst, const void *src, int64_t bytes, cudaStream_t s)
{
    if (bytes <= 0 || dst == src)
        return SSU_OK;
    return launch_kernel(copy_kernel, grid_for(bytes), kPoolThreads, 0, s,
                         static_cast<uint8_t *>(dst), static_cast<const uint8_t *>(src), bytes);
}

}  // namespace ssu
