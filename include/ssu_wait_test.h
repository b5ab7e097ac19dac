/*
 * ssu_wait_test.h -- the one extra entry point of the test library libssu_waittest.so.
 *
 * libssu_waittest.so is libssu.so built from the same sources with SSU_WAIT_TEST defined;
 * it exports every entry point of ssu.h plus the call below, and exists only so that the
 * test suite can make a kernel's bounded wait run out on purpose and check what happens
 * then (the kernel gives up, sets SSU_FLAG_TIMEOUT in err_flags, waits for its own copies
 * in flight, frees what it holds and returns; the context stays usable). The product
 * library libssu.so has neither this entry point nor the hooks behind it. No page the
 * library follows has a counterpart: this is test infrastructure.
 */
#ifndef SSU_WAIT_TEST_H
#define SSU_WAIT_TEST_H

#ifdef __cplusplus
extern "C" {
#endif

/* Which bounded wait a test can make run out (site argument). */
enum {
    SSU_WAIT_NONE = 0,
    SSU_WAIT_STREAM = 1,      /* a state tile of the per-warp streaming pipeline (decode,
                                 replay, fused conv decode, GDN decode); index = the tile's
                                 number in the chosen warp's sequence */
    SSU_WAIT_PREFILL = 2,     /* prefill chunk `index`: in the CUDA-core form its staged
                                 inputs, in the chunked tensor-core form its first MMAs
                                 (then not issued at all) */
    SSU_WAIT_TREE_STATE = 3,  /* the committed-state rows of a tree-verify item (tensor-core
                                 form); index = the item's position in its CTA's range */
    SSU_WAIT_TREE_X = 4,      /* the x tile of such an item */
    SSU_WAIT_TREE_MMA = 5     /* the MMA completion of such an item (its MMAs are then not
                                 issued at all) */
};

/*
 * ssu_test_wait_fault -- arm (or, with site SSU_WAIT_NONE, disarm) one wait of the next
 * launches on the current device, and set the limit of every bounded wait to limit_ns
 * nanoseconds (the product library's limit is 2 s).
 *   block  blockIdx.x of the CTA whose wait runs out
 *   warp   warp of that CTA (SSU_WAIT_STREAM; -1 matches every warp)
 *   index  which instance of the wait, counted within that CTA (or warp)
 * The chosen barrier is armed for 16 bytes more than its copies bring (for
 * SSU_WAIT_TREE_MMA: its MMAs and their commit are skipped), so every copy lands but the
 * wait cannot complete. The setting stays until the next call. Synchronous (it copies a
 * small record to device memory); not for use under stream capture.
 * Returns SSU_OK, SSU_ERR_SHAPE for limit_ns == 0, or SSU_ERR_CUDA.
 */
int ssu_test_wait_fault(int site, int block, int warp, int index,
                        unsigned long long limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* SSU_WAIT_TEST_H */
