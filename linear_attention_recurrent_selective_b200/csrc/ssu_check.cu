// ssu_check.cu -- debug check of the row-to-slot map.
//
// The padding contract of the FlashInfer page flashinfer.gdn_fused_decode_step
// (state_indices): each batch row reads and writes its own pool slot, a negative index is
// a padding row. Two active rows naming one slot would race, so the kernels take
// distinct indices as a precondition; this check, meant for debugging, reports what the
// kernels do not look for: two active rows with the same non-negative index
// (SSU_FLAG_DUPLICATE_INDEX) and an index >= P (SSU_FLAG_INDEX_RANGE).
//
// Thread i compares row i's index with the indices of every later row, which a block
// reads tile by tile into shared memory: O(active^2) comparisons (about 33 million at
// 8192 rows), no scratch memory, no host synchronisation.
#include "ssu_common.cuh"

namespace ssu {
namespace {

constexpr int kCheckThreads = 256;

__global__ void __launch_bounds__(kCheckThreads)
check_indices_kernel(const int32_t *idx, int32_t active, int32_t P, int32_t *err)
{
    __shared__ int32_t tile[kCheckThreads];
    const int i = blockIdx.x * kCheckThreads + threadIdx.x;
    const int32_t mine = i < active ? idx[i] : -1;
    int flags = mine >= P ? SSU_FLAG_INDEX_RANGE : 0;
    for (int j0 = blockIdx.x * kCheckThreads; j0 < active; j0 += kCheckThreads) {
        __syncthreads();                       // the previous tile has been read
        const int j = j0 + threadIdx.x;
        tile[threadIdx.x] = j < active ? idx[j] : -1;
        __syncthreads();
        if (mine >= 0) {
            const int n = min(kCheckThreads, active - j0);
            for (int k = 0; k < n; ++k)
                if (j0 + k > i && tile[k] == mine)
                    flags |= SSU_FLAG_DUPLICATE_INDEX;
        }
    }
    if (flags)
        atomicOr(err, flags);
}

}  // namespace

int launch_check_indices(const int32_t *idx, int32_t active, int32_t P, int32_t *err,
                         cudaStream_t s)
{
    const unsigned blocks = (unsigned)((active + kCheckThreads - 1) / kCheckThreads);
    return launch_kernel(check_indices_kernel, blocks, kCheckThreads, 0, s, idx, active, P, err);
}

}  // namespace ssu
