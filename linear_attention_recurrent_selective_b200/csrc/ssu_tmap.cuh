// ssu_tmap.cuh -- tensor (tiled) TMA copies of node-row tiles, sm_100a inline PTX.
//
// A tensor of rows x H x Dm elements (x or out of the tree verify: rows = batch x nodes) is
// described to the Tensor Memory Accelerator once per launch by a tensor map; one
// instruction then moves a whole tile of (128 bytes of dims) x (one head) x (box rows)
// between global and shared memory, however strided the rows are in global memory. In
// shared memory the box is dense, 128 bytes per row, with the 128-byte swizzle: the
// 16-byte chunk c of row r of a 1024-byte aligned box sits at chunk position c ^ (r % 8).
// Loads complete on an mbarrier's transaction count; elements outside the tensor read as
// zero and are not written by stores. No multicast form is used.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "ssu_async.cuh"

namespace ssu {

// The driver's cuTensorMapEncodeTiled, looked up once per process (null when missing).
inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map over t[rows][H][Dm] of `dtype` (SSU_F32, SSU_F16 or SSU_BF16) with a box of
// 128 bytes of dims x 1 head x box_rows rows, 128-byte swizzle, zero fill. False when the
// tensor cannot be described that way: base not 16-byte aligned, a row of dims not a
// multiple of 16 bytes or shorter than the box, box_rows outside 1 .. 256, or no encoder.
inline bool encode_rows_map(CUtensorMap *m, const void *base, int dtype, int64_t Dm, int64_t H,
                            int64_t rows, int box_rows)
{
    const int es = dtype == SSU_F32 ? 4 : 2;
    const CUtensorMapDataType t = dtype == SSU_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                  : dtype == SSU_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                     : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int box_dims = 128 / es;
    if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (Dm * es) % 16 != 0 || Dm < box_dims ||
        box_rows < 1 || box_rows > 256 || rows < 1 || H < 1 || rows > (int64_t)UINT32_MAX)
        return false;
    PFN_cuTensorMapEncodeTiled_v12000 enc = tmap_encoder();
    if (!enc)
        return false;
    const cuuint64_t dims[3] = {(cuuint64_t)Dm, (cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)(Dm * es), (cuuint64_t)(H * Dm * es)};
    const cuuint32_t box[3] = {(cuuint32_t)box_dims, 1u, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(m, t, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tile load: dims d .. d + 128 / es - 1 of head h, rows r .. r + box_rows - 1, into
// dst (1024-byte aligned), completing its box bytes on bar.
__device__ __forceinline__ void tma_load_rows(void *dst, const CUtensorMap *map, int d, int h,
                                              int r, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(d), "r"(h), "r"(r),
        "r"(smem_u32(bar))
        : "memory");
}

// Tile store of the same box from src (1024-byte aligned) into the tensor; elements
// outside it are not written. Tracked by this thread's bulk async-groups.
__device__ __forceinline__ void tma_store_rows(const CUtensorMap *map, const void *src, int d,
                                               int h, int r)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(d), "r"(h),
                 "r"(r)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// This thread's committed stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all()
{
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// This thread's committed stores are complete.
__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace ssu
