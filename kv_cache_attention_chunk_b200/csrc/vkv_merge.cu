// vkv_lse_merge: exact recombination of two partial attentions by their LSE
// (ISPA summary, section 2 step 1 "Dual-Stream Warmup" and contribution 2:
// branch outputs tracked with their log-sum-exp, merged by online softmax).
//
// Bandwidth-bound: every output row reads 2 x d bf16 + 2 fp32 and writes
// d bf16 + 1 fp32.  One thread handles 8 features (one 16-byte vector) of a
// row; consecutive threads cover consecutive 16-byte chunks of the
// [B, Lq, H, d] tensors, so loads and stores are fully coalesced.
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

__global__ void __launch_bounds__(256) lse_merge_kernel(const MergeParams p) {
  const int cpr = p.d >> 3;  // 16-byte chunks per row
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < p.n_chunks;
       t += (long long)gridDim.x * blockDim.x) {
    const long long row = t / cpr;
    const int ch = (int)(t - row * cpr);
    const int h = (int)(row % p.H);
    const long long bi = row / p.H;
    const int i = (int)(bi % p.Lq);
    const int b = (int)(bi / p.Lq);
    const size_t li = ((size_t)b * p.H + h) * p.Lq + i;
    const float la = __ldg(p.la + li);
    const float lb = __ldg(p.lb + li);
    const float M = fmaxf(la, lb);
    const bool empty = (M == -INFINITY);
    const float Ms = empty ? 0.f : M;
    constexpr float kLog2e = 1.4426950408889634f;
    const float wa = ex2_approx((la - Ms) * kLog2e);
    const float wb = ex2_approx((lb - Ms) * kLog2e);
    const float den = wa + wb;
    const float ca = empty ? 0.f : wa / den;
    const float cb = empty ? 0.f : wb / den;
    const uint4 va = __ldcs(reinterpret_cast<const uint4*>(p.oa + b * p.a_sb + (long long)i * p.a_st +
                                                            h * p.a_sh) + ch);
    const uint4 vb = __ldcs(reinterpret_cast<const uint4*>(p.ob + b * p.b_sb + (long long)i * p.b_st +
                                                            h * p.b_sh) + ch);
    const uint32_t xa[4] = {va.x, va.y, va.z, va.w};
    const uint32_t xb[4] = {vb.x, vb.y, vb.z, vb.w};
    uint32_t r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a0 = __uint_as_float(xa[e] << 16), a1 = __uint_as_float(xa[e] & 0xFFFF0000u);
      const float b0 = __uint_as_float(xb[e] << 16), b1 = __uint_as_float(xb[e] & 0xFFFF0000u);
      r[e] = pack_bf16x2(ca * a0 + cb * b0, ca * a1 + cb * b1);
    }
    __stcs(reinterpret_cast<uint4*>(p.oo + b * p.o_sb + (long long)i * p.o_st + h * p.o_sh) + ch,
           make_uint4(r[0], r[1], r[2], r[3]));
    if (ch == 0) p.lo[li] = empty ? -INFINITY : Ms + lg2_approx(den) * 0.6931471805599453f;
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
  if (d <= 0 || d % 8 != 0 || d > 1024) return VKV_ERR_UNSUPPORTED;
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
  const long long want = (p.n_chunks + 255) / 256;
  const int grid = (int)std::min<long long>(want, (long long)n_sm * 16);
  lse_merge_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  return VKV_OK;
}
