// vkv_lse_merge: exact recombination of two partial attentions by their LSE
// (ISPA summary, section 2 step 1 "Dual-Stream Warmup" and contribution 2:
// branch outputs tracked with their log-sum-exp, merged by online softmax).
//
// Bandwidth-bound: every output row reads 2 x d bf16 + 2 fp32 and writes
// d bf16 + 1 fp32.  A thread handles 16-byte chunks (8 features) of rows;
// consecutive threads cover consecutive chunks of the [B, Lq, H, d] tensors,
// so loads and stores are fully coalesced.
#include "vkv_internal.h"
#include "vkv_ptx.cuh"

namespace vkv {
namespace {

struct MergeParams {
  const __nv_bfloat16* oa;
  const __nv_bfloat16* ob;
  __nv_bfloat16* oo;
  long long a_sb, a_st, a_sh, b_sb, b_st, b_sh, o_sb, o_st, o_sh;
  const float* la;
  const float* lb;
  float* lo;
  int B, H, Lq, d;
  long long n_chunks;  // B * Lq * H * (d / 8)
};

#ifndef VKV_MERGE_POS
#define VKV_MERGE_POS 4
#endif
constexpr int kMergePos = VKV_MERGE_POS;  // consecutive (b, i) query positions per thread

// grid: x = ceil(B * Lq / kMergePos) position groups, y = column blocks of at
// most 256 threads (H * d/8 columns split as evenly as whole warps allow).
// Thread: one 16-byte column (head h, chunk ch) of kMergePos consecutive query
// positions; all its loads are issued before the first merge, and the index
// of the next position is advanced without division.  The output may alias an
// input (in-place merge): each chunk is read before it is written, by the same
// thread.
template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(const MergeParams p) {
  constexpr int CPR = D / 8;
  const int col = blockIdx.y * blockDim.x + threadIdx.x;
  if (col >= p.H * CPR) return;
  const int h = col / CPR, ch = col % CPR;
  const int pos0 = blockIdx.x * kMergePos;
  const int n_pos = p.B * p.Lq;
  int b = pos0 / p.Lq, i = pos0 - (pos0 / p.Lq) * p.Lq;
  uint4 va[kMergePos], vb[kMergePos];
  float la[kMergePos], lb[kMergePos];
  int bb[kMergePos], ii[kMergePos];
#pragma unroll
  for (int k = 0; k < kMergePos; ++k) {
    bb[k] = b;
    ii[k] = i;
    if (pos0 + k < n_pos) {
      const size_t li = ((size_t)b * p.H + h) * p.Lq + i;
      va[k] = __ldcs(reinterpret_cast<const uint4*>(p.oa + b * p.a_sb + (long long)i * p.a_st + h * p.a_sh) + ch);
      vb[k] = __ldcs(reinterpret_cast<const uint4*>(p.ob + b * p.b_sb + (long long)i * p.b_st + h * p.b_sh) + ch);
      la[k] = __ldg(p.la + li);
      lb[k] = __ldg(p.lb + li);
    }
    if (++i == p.Lq) {
      i = 0;
      ++b;
    }
  }
  constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
  for (int k = 0; k < kMergePos; ++k) {
    if (pos0 + k >= n_pos) break;
    const float M = fmaxf(la[k], lb[k]);
    const bool empty = (M == -INFINITY);
    const float Ms = empty ? 0.f : M;
    const float wa = ex2_approx((la[k] - Ms) * kLog2e);
    const float wb = ex2_approx((lb[k] - Ms) * kLog2e);
    const float den = wa + wb;
    const float ca = empty ? 0.f : wa / den;
    const float cb = empty ? 0.f : wb / den;
    const uint32_t xa[4] = {va[k].x, va[k].y, va[k].z, va[k].w};
    const uint32_t xb[4] = {vb[k].x, vb[k].y, vb[k].z, vb[k].w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a0 = __uint_as_float(xa[e] << 16), a1 = __uint_as_float(xa[e] & 0xFFFF0000u);
      const float b0 = __uint_as_float(xb[e] << 16), b1 = __uint_as_float(xb[e] & 0xFFFF0000u);
      o[e] = pack_bf16x2(ca * a0 + cb * b0, ca * a1 + cb * b1);
    }
    __stcs(reinterpret_cast<uint4*>(p.oo + bb[k] * p.o_sb + (long long)ii[k] * p.o_st + h * p.o_sh) + ch,
           make_uint4(o[0], o[1], o[2], o[3]));
    if (ch == 0)
      p.lo[((size_t)bb[k] * p.H + h) * p.Lq + ii[k]] =
          empty ? -INFINITY : Ms + lg2_approx(den) * 0.6931471805599453f;
  }
}

}  // namespace
}  // namespace vkv

using namespace vkv;

extern "C" vkv_status vkv_lse_merge(vkv_tensor o_a, const float* lse_a, vkv_tensor o_b, const float* lse_b,
                                    vkv_tensor o_out, float* lse_out, int32_t B, int32_t H, int32_t Lq,
                                    int32_t d, vkv_stream_t stream) {
  if (!o_a.ptr || !o_b.ptr || !o_out.ptr || !lse_a || !lse_b || !lse_out) return VKV_ERR_NULL;
  if (B <= 0 || H <= 0 || Lq <= 0) return VKV_ERR_SHAPE;
  if (d != 64 && d != 128) return VKV_ERR_UNSUPPORTED;
  if ((long long)B * Lq >= (1ll << 31) - kMergePos || (long long)H * (d / 8) >= (1ll << 31))
    return VKV_ERR_UNSUPPORTED;
  if (!tensor_aligned(o_a) || !tensor_aligned(o_b) || !tensor_aligned(o_out)) return VKV_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(lse_a) | reinterpret_cast<uintptr_t>(lse_b) |
       reinterpret_cast<uintptr_t>(lse_out)) & 3u)
    return VKV_ERR_ALIGN;
  int dev = 0;
  const int n_sm = device_sm_count(&dev);
  if (n_sm <= 0) return VKV_ERR_CUDA;
  MergeParams p;
  p.oa = reinterpret_cast<const __nv_bfloat16*>(o_a.ptr);
  p.ob = reinterpret_cast<const __nv_bfloat16*>(o_b.ptr);
  p.oo = reinterpret_cast<__nv_bfloat16*>(o_out.ptr);
  p.a_sb = o_a.sb; p.a_st = o_a.st; p.a_sh = o_a.sh;
  p.b_sb = o_b.sb; p.b_st = o_b.st; p.b_sh = o_b.sh;
  p.o_sb = o_out.sb; p.o_st = o_out.st; p.o_sh = o_out.sh;
  p.la = lse_a;
  p.lb = lse_b;
  p.lo = lse_out;
  p.B = B;
  p.H = H;
  p.Lq = Lq;
  p.d = d;
  p.n_chunks = (long long)B * Lq * H * (d / 8);
  const long long n_pos = (long long)B * Lq;
  // column blocks of at most 256 threads, as even as warps allow (few idle lanes)
  const int cols = H * (d / 8);
  const int n_cb = (cols + 255) / 256;
  const int width = (((cols + n_cb - 1) / n_cb) + 31) / 32 * 32;
  const dim3 grid((unsigned)((n_pos + kMergePos - 1) / kMergePos), (unsigned)n_cb);
  if (grid.y > 65535u) return VKV_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128)
    lse_merge_kernel<128><<<grid, width, 0, st>>>(p);
  else
    lse_merge_kernel<64><<<grid, width, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  return VKV_OK;
}
