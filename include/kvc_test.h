/*
 * kvc_test.h — test-only entry point of libkvc.so. Not part of the codec's
 * interface: it exists so that a test can make one of the codec's bounded
 * device waits run out, on purpose and harmlessly, and check that the call
 * ends with KVC_ERR_TIMEOUT while the CUDA context stays usable.
 *
 * Every wait of the codec's kernels is bounded (one second of the GPU's
 * global timer, or an iteration cap); when one runs out the kernel records
 * KVC_ERR_TIMEOUT in the workspace status word, every other wait of the call
 * sees it and gives up at once, and the kernels return. In a correct call no
 * wait runs out, so this path is otherwise unreachable.
 */
#ifndef KVC_TEST_H
#define KVC_TEST_H

#include "kvc.h"

#ifdef __cplusplus
extern "C" {
#endif

/* kvc_compress with two changes to its compaction kernel (which runs only
 * when code chunks are stored zero-byte eliminated): the kernel's tickets
 * start skip_chunks chunks after the first shrinking code chunk, so those
 * chunks are never read and their read flags never set; and its waits give
 * up after wait_ns nanoseconds instead of one second. The first chunk the
 * kernel does take stores into the slot of a skipped chunk, so its wait for
 * that chunk's read flag runs out: the call ends with KVC_ERR_TIMEOUT in the
 * status word (read it with kvc_stream_status) and an unspecified stream.
 * Writes stay inside [out, out + out_capacity) and the workspace.
 * Arguments as kvc_compress; skip_chunks >= 1; 0 < wait_ns <= 1e9, else
 * KVC_ERR_INVALID_ARG. Without code-region elimination (no shrinking code
 * chunk, or reading R16 stores every code chunk raw) the compaction does not
 * run and the call is an ordinary kvc_compress. */
kvc_status kvc_test_compress_stalled(const kvc_kv_desc *kv, const kvc_params *params,
                                     void *out, size_t out_capacity, uint64_t *out_bytes_dev,
                                     void *workspace, size_t workspace_bytes,
                                     uint32_t skip_chunks, uint64_t wait_ns,
                                     kvc_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* KVC_TEST_H */
