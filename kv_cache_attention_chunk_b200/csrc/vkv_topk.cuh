// Exact top-K of one query block's window-block scores, computed by one warp
// (Sparse Forcing summary, section 2 component 3 "PBSA": each query block
// attends to the K window blocks whose representatives score highest).  Used
// by the standalone selection kernel and by the block-sparse attention kernel
// when it selects for itself, so both make the same choice.
#pragma once

#include <stdint.h>

namespace vkv {

// A block score as it is ranked: NaN ranks last (as -inf) and -0 counts as +0,
// so equal scores tie and fall back to the block index.
__device__ __forceinline__ float rank_score(float v) { return (v != v) ? -INFINITY : (v == 0.f ? 0.f : v); }

// Order-preserving 32-bit image of a ranked score (larger score, larger key).
__device__ __forceinline__ uint32_t score_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return u ^ ((u >> 31) ? 0xFFFFFFFFu : 0x80000000u);
}

// The topk (1 <= topk <= n) largest of the n keys kq[0..n) (shared memory),
// ties to the lower index, by all 32 lanes of one warp with warp barriers only.
// Radix selection of the K-th largest key, 8 bits a pass (4 passes): the keys
// still in play (those that share the threshold's digits found so far) are
// counted per digit in the warp's histogram hq[256] (shared memory), one atomic
// per distinct digit and chunk of 32 keys; the lanes scan it from the top and
// fix the next digit where the running count reaches the number still to take.
// Then, in ascending index order, every key above the threshold is kept, and of
// the keys equal to it the lowest indices, as many as are still to take.
// out (optional): the kept indices, ascending, topk of them.
// words (optional): bit i of words[c] is set when index 32c + i is kept.
__device__ __forceinline__ void warp_topk(const uint32_t* kq, int n, int topk, int* hq, int* out,
                                          uint32_t* words) {
  const int lane = (int)(threadIdx.x & 31u);
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t thr = 0u;
  int need = topk;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
#pragma unroll
    for (int i = 0; i < 8; ++i) hq[lane + 32 * i] = 0;
    __syncwarp();
    for (int w0 = 0; w0 < n; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t k = w < n ? kq[w] : 0u;
      const bool in_play = w < n && (k & hi_mask) == thr;
      const uint32_t digit = in_play ? ((k >> shift) & 255u) : 0xFFFFFFFFu;
      const unsigned grp = __match_any_sync(0xFFFFFFFFu, digit);
      if (in_play && (grp & lt) == 0u) atomicAdd(&hq[digit], __popc(grp));
    }
    __syncwarp();
    // lane l holds digits 255 - 8l .. 248 - 8l (lane 0 the largest)
    int cnt[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cnt[i] = hq[255 - (8 * lane + i)];
      sum += cnt[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += t;
    }
    int above = incl - sum;  // keys in play with a digit above this lane's bins
    const bool mine = above < need && need <= incl;
    uint32_t digit = 0u;
    int rest = 0;
    if (mine) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (above + cnt[i] >= need) {
          digit = (uint32_t)(255 - (8 * lane + i));
          rest = need - above;
          break;
        }
        above += cnt[i];
      }
    }
    const int src = __ffs(__ballot_sync(0xFFFFFFFFu, mine)) - 1;
    thr |= __shfl_sync(0xFFFFFFFFu, digit, src) << shift;
    need = __shfl_sync(0xFFFFFFFFu, rest, src);
    __syncwarp();  // the histogram is read before the next pass clears it
  }
  // keys above the threshold, then the lowest-index keys equal to it, in ascending order
  int written = 0, eq_seen = 0;
  for (int w0 = 0; w0 < n; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t k = w < n ? kq[w] : 0u;
    const bool valid = w < n;
    const bool eq = valid && k == thr;
    const uint32_t beq = __ballot_sync(0xFFFFFFFFu, eq);
    const bool keep = valid && (k > thr || (eq && eq_seen + __popc(beq & lt) < need));
    eq_seen += __popc(beq);
    const uint32_t bk = __ballot_sync(0xFFFFFFFFu, keep);
    if (out && keep) out[written + __popc(bk & lt)] = w;
    if (words && lane == 0) words[w0 >> 5] = bk;
    written += __popc(bk);
  }
}

}  // namespace vkv
