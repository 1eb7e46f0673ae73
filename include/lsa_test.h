/*
 * lsa_test.h -- test-only switches of liblsa_test.so.
 *
 * liblsa_test.so is built from the same sources as liblsa.so, with one extra
 * entry point.  The product library liblsa.so does not export it and has no
 * switch of any kind (no environment variable is read): a serving process
 * cannot change its kernel path or break its handoffs by accident.  Tests load
 * liblsa_test.so when they need one of the switches below, and liblsa.so
 * otherwise.  The paper has no counterpart of this file.
 */
#ifndef LSA_TEST_H_
#define LSA_TEST_H_

#include "lsa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Sets the switches for every later call into liblsa_test.so in this process
 * (process-wide, not thread-safe: set them before the calls they affect).
 *   force_simt_path        != 0: every call runs the CUDA-core kernels instead
 *                          of the tensor-core ones (to compare the two GPU
 *                          paths on the same inputs); 0: the normal choice.
 *   split_select_min_cols  rows of at least this many positions take the split
 *                          select inside lsa_decode_step; < 0: the library's
 *                          default (2^18).
 *   scan_wait_extra        added to the count of scan CTAs that the decode
 *                          step's top-k waits for.  Any value > 0 makes that
 *                          count unreachable, so the top-k's bounded wait and
 *                          then the attention's run out after about a second
 *                          each and record LSA_ERR_TIMEOUT in the status word
 *                          (the failure path of the handoff, without a fault).
 *   no_cluster_topk        != 0: rows of up to 2^18 positions take the collect
 *                          + per-row select top-k instead of the
 *                          one-cluster-per-row kernel (to compare the two).
 * Returns LSA_OK.
 */
lsa_status lsa_test_set_hooks(int32_t force_simt_path, int64_t split_select_min_cols, uint32_t scan_wait_extra,
                              int32_t no_cluster_topk);

/*
 * The decode scan's tile schedule inside lsa_decode_step and the DSA order of
 * lsa_decode_layers, for every later call in this process (process-wide, not
 * thread-safe).  With a pool, each scan CTA first takes its even share of the
 * first static_pm thousandths of the tiles, then claims chunks of `chunk`
 * tiles from a counter until none is left.
 *   static_pm  0 .. 1000; > 1000: no pool (every tile in the static shares);
 *              < 0: the library's default (no pool).
 *   chunk      tiles per claim; <= 0: the default (4).
 * Every schedule computes each tile the same way, so the results are bitwise
 * the same; tests compare them.  Returns LSA_OK.
 */
lsa_status lsa_test_set_scan_pool(int32_t static_pm, int32_t chunk);

#ifdef __cplusplus
}
#endif

#endif /* LSA_TEST_H_ */
