// vkv_compact_cache: head-aware cache compaction into a flattened ragged cache
// (Pyramid Forcing summary, methodology section 2: per-head-type cache policies
// sharing the sink and the forced recent frames -- adaptive-stride anchors,
// period-P waves, pairwise-merged veils; section 3: variable-length caches
// stored as flattened sequences with boundary indices, packed in one launch).
//
// The host expands each head's rule into a list of stored pieces (a source
// frame, or a pair of adjacent source frames to merge), in output order, and
// passes the piece table and the boundary offsets as kernel parameters.  The
// kernel is a pure HBM stream: CTA (piece, 64-row block, tensor) copies 64 rows
// of d bf16 with 16-byte loads and stores, averaging the two source rows of a
// merged piece in fp32 and rounding to nearest-even bf16.
#include <cstring>
#include <memory>
#include <vector>

#include "vkv_internal.h"
#include "vkv_ptx.cuh"

namespace vkv {
namespace {

struct Piece {
  int out_row0;  // first output row
  int f0, f1;    // source frame(s); f1 < 0: plain copy
  int seq;       // b*H + h
};

struct CompactParams {
  const __nv_bfloat16* src[2];
  __nv_bfloat16* dst[2];
  long long sb[2], st[2], sh[2];
  int H, d, frame_tokens, blocks_per_piece, n_seq;
  int* cu_dev;
  int cu[VKV_COMPACT_MAX_SEQS + 1];
  Piece pieces[VKV_COMPACT_MAX_PIECES];
};

constexpr int kCompactRows = 64;  // rows per CTA

// grid: x = n_pieces * blocks_per_piece, y = 2 (K, V); 256 threads.
template <int D>
__global__ void __launch_bounds__(256) compact_kernel(const __grid_constant__ CompactParams p) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  const int pi = blockIdx.x / p.blocks_per_piece;
  const int rb = blockIdx.x - pi * p.blocks_per_piece;
  const int tsr = blockIdx.y;
  if (blockIdx.x == 0 && tsr == 0)
    for (int i = threadIdx.x; i <= p.n_seq; i += blockDim.x) p.cu_dev[i] = p.cu[i];
  const Piece pc = p.pieces[pi];
  const int b = pc.seq / p.H, h = pc.seq - (pc.seq / p.H) * p.H;
  const int t0 = rb * kCompactRows;
  const int nrows = min(kCompactRows, p.frame_tokens - t0);
  const __nv_bfloat16* base = p.src[tsr] + b * p.sb[tsr] + h * p.sh[tsr];
  __nv_bfloat16* out = p.dst[tsr] + (long long)(pc.out_row0 + t0) * D;
  const bool merge = pc.f1 >= 0;
  const long long r0 = (long long)pc.f0 * p.frame_tokens + t0;
  const long long r1 = (long long)pc.f1 * p.frame_tokens + t0;
  constexpr int PER = kCompactRows * CPR / 256;  // chunks per thread
  uint4 a[PER], c[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * 256;
    const int row = i / CPR, ch = i - (i / CPR) * CPR;
    if (row < nrows) {
      a[k] = __ldcs(reinterpret_cast<const uint4*>(base + (r0 + row) * p.st[tsr]) + ch);
      if (merge) c[k] = __ldcs(reinterpret_cast<const uint4*>(base + (r1 + row) * p.st[tsr]) + ch);
    }
  }
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * 256;
    const int row = i / CPR, ch = i - (i / CPR) * CPR;
    if (row >= nrows) continue;
    uint4 o = a[k];
    if (merge) {
      const uint32_t xa[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
      const uint32_t xc[4] = {c[k].x, c[k].y, c[k].z, c[k].w};
      uint32_t m[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // the fp32 sum of two bf16 values is exact, and so is halving it
        const float lo = (__uint_as_float(xa[e] << 16) + __uint_as_float(xc[e] << 16)) * 0.5f;
        const float hi = (__uint_as_float(xa[e] & 0xFFFF0000u) + __uint_as_float(xc[e] & 0xFFFF0000u)) * 0.5f;
        m[e] = pack_bf16x2(lo, hi);
      }
      o = make_uint4(m[0], m[1], m[2], m[3]);
    }
    __stcs(reinterpret_cast<uint4*>(out + (long long)row * D) + ch, o);
  }
}

// Stored pieces of one head, in output order: (f0, f1), f1 = -1 for a single frame.
bool head_pieces(const vkv_compact_args* a, const vkv_head_rule& r, std::vector<std::pair<int, int>>* out) {
  const int lo = 1, hi = a->hist_frames - a->recent_frames - 1;
  const int n_mid = hi >= lo ? hi - lo + 1 : 0;
  out->clear();
  out->push_back({0, -1});
  switch (r.policy) {
    case VKV_HEAD_FULL:
      for (int f = lo; f <= hi; ++f) out->push_back({f, -1});
      break;
    case VKV_HEAD_ANCHOR:
      if (r.param < 1 || r.param > n_mid) return false;
      if (r.param == 1) {
        out->push_back({lo, -1});
      } else {
        for (int i = 0; i < r.param; ++i) {
          // floor of the evenly spaced position, in exact integer arithmetic
          const long long num = (long long)i * (hi - lo);
          out->push_back({lo + (int)(num / (r.param - 1)), -1});
        }
      }
      break;
    case VKV_HEAD_WAVE:
      if (r.param < 1) return false;
      for (int f = lo; f <= hi; ++f)
        if ((a->hist_frames - f) % r.param == 0) out->push_back({f, -1});
      break;
    case VKV_HEAD_VEIL:
      if (r.param < 0 || (r.param & 1) || r.param > n_mid) return false;
      for (int f = hi - r.param + 1; f <= hi; f += 2) out->push_back({f, f + 1});
      break;
    default:
      return false;
  }
  for (int f = a->hist_frames - a->recent_frames; f < a->hist_frames; ++f) out->push_back({f, -1});
  for (int f = a->hist_frames; f < a->hist_frames + a->cur_frames; ++f) out->push_back({f, -1});
  return true;
}

// Validates the sizes and rules; fills the piece table and offsets when asked.
vkv_status plan_compact(const vkv_compact_args* a, std::vector<Piece>* pieces, std::vector<long long>* cu) {
  if (!a) return VKV_ERR_NULL;
  if (a->B <= 0 || a->H <= 0 || a->frame_tokens <= 0 || a->hist_frames < 1 || a->cur_frames < 0 ||
      a->recent_frames < 0 || a->hist_frames < 1 + a->recent_frames)
    return VKV_ERR_SHAPE;
  if (a->d != 64 && a->d != 128) return VKV_ERR_UNSUPPORTED;
  if (!a->rules) return VKV_ERR_NULL;
  const long long n_seq = (long long)a->B * a->H;
  std::vector<std::pair<int, int>> hp;
  long long rows = 0;
  if (cu) cu->assign(1, 0);
  for (int b = 0; b < a->B; ++b) {
    for (int h = 0; h < a->H; ++h) {
      if (!head_pieces(a, a->rules[h], &hp)) return VKV_ERR_SHAPE;
      if (rows + (long long)hp.size() * a->frame_tokens >= (1ll << 31)) return VKV_ERR_UNSUPPORTED;
      for (const auto& pp : hp) {
        if (pieces) pieces->push_back({(int)rows, pp.first, pp.second, b * a->H + h});
        rows += a->frame_tokens;
      }
      if (cu) cu->push_back(rows);
    }
  }
  if (pieces && (n_seq > VKV_COMPACT_MAX_SEQS || (long long)pieces->size() > VKV_COMPACT_MAX_PIECES))
    return VKV_ERR_UNSUPPORTED;
  return VKV_OK;
}

}  // namespace
}  // namespace vkv

using namespace vkv;

extern "C" int64_t vkv_compact_rows(const vkv_compact_args* a) {
  std::vector<long long> cu;
  const vkv_status st = plan_compact(a, nullptr, &cu);
  if (st != VKV_OK) return -(int64_t)st;
  return (int64_t)cu.back();
}

extern "C" vkv_status vkv_compact_cache(const vkv_compact_args* a, vkv_stream_t stream) {
  std::vector<Piece> pieces;
  std::vector<long long> cu;
  const vkv_status st = plan_compact(a, &pieces, &cu);
  if (st != VKV_OK) return st;
  if (!a->k_src.ptr || !a->v_src.ptr || !a->k_out || !a->v_out || !a->cu_seqlens) return VKV_ERR_NULL;
  if (!tensor_aligned(a->k_src) || !tensor_aligned(a->v_src)) return VKV_ERR_ALIGN;
  if (((reinterpret_cast<uintptr_t>(a->k_out) | reinterpret_cast<uintptr_t>(a->v_out)) & 15u) ||
      (reinterpret_cast<uintptr_t>(a->cu_seqlens) & 3u))
    return VKV_ERR_ALIGN;
  if (cu.back() > a->out_rows) return VKV_ERR_RANGE;
  const long long n_seq = (long long)a->B * a->H;
  if (a->cu_seqlens_host)
    for (long long i = 0; i <= n_seq; ++i) a->cu_seqlens_host[i] = (int32_t)cu[i];
  if (pieces.empty()) return VKV_OK;
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  auto P = std::make_unique<CompactParams>();
  std::memset(P.get(), 0, sizeof(CompactParams));
  const vkv_tensor* srcs[2] = {&a->k_src, &a->v_src};
  void* dsts[2] = {a->k_out, a->v_out};
  for (int i = 0; i < 2; ++i) {
    P->src[i] = reinterpret_cast<const __nv_bfloat16*>(srcs[i]->ptr);
    P->dst[i] = reinterpret_cast<__nv_bfloat16*>(dsts[i]);
    P->sb[i] = srcs[i]->sb;
    P->st[i] = srcs[i]->st;
    P->sh[i] = srcs[i]->sh;
  }
  P->H = a->H;
  P->d = a->d;
  P->frame_tokens = a->frame_tokens;
  P->blocks_per_piece = (a->frame_tokens + kCompactRows - 1) / kCompactRows;
  P->n_seq = (int)n_seq;
  P->cu_dev = a->cu_seqlens;
  for (long long i = 0; i <= n_seq; ++i) P->cu[i] = (int)cu[i];
  for (size_t i = 0; i < pieces.size(); ++i) P->pieces[i] = pieces[i];
  const long long nblk = (long long)pieces.size() * P->blocks_per_piece;
  if (nblk > 0x7FFFFFFFll) return VKV_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)nblk, 2);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (a->d == 128)
    compact_kernel<128><<<grid, 256, 0, s>>>(*P);
  else
    compact_kernel<64><<<grid, 256, 0, s>>>(*P);
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  return VKV_OK;
}
