/*
 * vkv_test.h -- test aids of the chunk-attention library.
 *
 * These entry points exist only in the test build of the library
 * (libvkv_test.so, compiled with VKV_TEST_AIDS defined); the production
 * library libvkv.so neither exports them nor carries the code paths they
 * switch on.  Everything in vkv.h is exported by both builds.
 */
#ifndef VKV_TEST_H_
#define VKV_TEST_H_

#include "vkv.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * vkv_debug_withhold_copy -- test aid for the bounded pipeline waits.  The next
 * n_calls launches of vkv_chunk_attn or vkv_latent_attn (in any thread of the
 * process) run with the first cache-tile copy of every CTA withheld: the wait
 * for it runs out after its time limit (1 s), the kernel stops its work, lets
 * the copies it did issue land, releases its resources and writes
 * VKV_DEVERR_TIMEOUT to err_word; the outputs of that launch are incomplete and
 * the device stays usable.  n_calls = 0 disarms it.  Returns VKV_ERR_SHAPE for
 * n_calls < 0.  Process-global: a concurrent caller's launches may take the
 * armed calls, which is why it lives only in the test build.
 */
vkv_status vkv_debug_withhold_copy(int32_t n_calls);

/*
 * vkv_debug_exp2_poly -- test aid: y[i] = the attention softmax's FMA-pipe 2^x
 * (range reduction to [-1/2, 1/2] and a cubic minimax polynomial, used for part
 * of the score columns) for n DEVICE fp32 values x (n >= 1), asynchronous on
 * `stream`.  Lets a test compare the device function with 2^x.
 */
vkv_status vkv_debug_exp2_poly(const float* x, float* y, int32_t n, vkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* VKV_TEST_H_ */
