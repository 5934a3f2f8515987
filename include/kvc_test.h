/*
 * kvc_test.h — test-only entry points of libkvc.so. Not part of the codec's
 * interface: one exists so that a test can make one of the codec's bounded
 * device waits run out, on purpose and harmlessly, and check that the call
 * ends with KVC_ERR_TIMEOUT while the CUDA context stays usable; the other
 * runs the FP4 quantizer's device rounding on given values so that a test
 * can compare it with the rule it implements at every tie.
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

/* The FP4 quantizer's e2m1 rounding (the same device function its encoder
 * uses) on n DEVICE fp32 values: out[i] = the e2m1 code nearest to in[i],
 * ties to the even magnitude index, magnitudes above 6 to 6, magnitude 0
 * always code 0 (no negative zero). in, out: device pointers; n < 2^31,
 * else KVC_ERR_INVALID_ARG. Asynchronous on `stream`. */
kvc_status kvc_test_e2m1(const float *in, uint8_t *out, uint64_t n, kvc_stream_t stream);

/* The quantizers' division by their constant (the same device function the
 * encoder uses for fl(x / (2^b - 1)) and fl(x / (2^(b-1) - 1))) on n DEVICE
 * fp32 values x >= 0: out[i] = in[i] / q rounded to nearest even, for q in
 * {1, 3, 7, 15, 127, 255} (else KVC_ERR_INVALID_ARG; n < 2^31).
 * Asynchronous on `stream`. */
kvc_status kvc_test_div_const(const float *in, float *out, uint64_t n, int q,
                              kvc_stream_t stream);

/* The encoder's reciprocal of its stored scales (the same device function it
 * uses for 1 / s, s = an fp16 scale times 2^K) on n DEVICE fp32 values:
 * out[i] = 1 / in[i] rounded to nearest even, for in[i] a positive finite
 * fp16 value times 8 or 16 (other inputs: the result is not specified);
 * n < 2^31, else KVC_ERR_INVALID_ARG. Asynchronous on `stream`. */
kvc_status kvc_test_rcp_scale(const float *in, float *out, uint64_t n, kvc_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* KVC_TEST_H */
