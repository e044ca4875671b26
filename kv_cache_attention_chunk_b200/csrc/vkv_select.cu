// vkv_block_select: blockified coarse scoring and top-K window-block selection
// (Sparse Forcing summary, section 2 component 2 "Blockified Compression": one
// representative token per block for coarse scoring; component 3 "PBSA":
// top-K blocks of the local window, per query block).
//
// Two kernels on the caller's stream:
//   pool_kernel     mean of every 64-row block of Q and of the window part of K,
//                   in fp32, written to the caller's workspace.  One CTA of 128
//                   threads per (block, batch*head): 16 threads cover a 256-byte
//                   row with 16-byte loads, 8 row groups of 8 rows each; the
//                   groups are combined in shared memory.  HBM-bound.
//   select_kernel   one warp per (batch*head, query block): scores against every
//                   window block (coalesced reads of the pooled keys, warp
//                   reduction), then an exact rank-based top-K: block w is kept
//                   iff fewer than K blocks beat it (higher score, or equal score
//                   and lower index); kept blocks are written in ascending order.
#include <algorithm>
#include <mutex>

#include "vkv_internal.h"
#include "vkv_ptx.cuh"

namespace vkv {
namespace {

struct PoolParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  long long q_sb, q_st, q_sh, k_sb, k_st, k_sh;
  int B, H, d, Lq, n_qblk, n_win, win_row0;
  float* qbar;  // [B*H][n_qblk][d]
  float* kbar;  // [B*H][n_win][d]
};

// grid: x = block index over n_qblk + n_win, y = b*H + h; 128 threads.
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const PoolParams p) {
  constexpr int CPR = D / 8;        // 16-byte chunks per row
  constexpr int GROUPS = 128 / CPR;  // row groups
  constexpr int RPG = 64 / GROUPS;   // rows per group
  __shared__ float part[GROUPS][D];
  const int blk = blockIdx.x;
  const int s = blockIdx.y;
  const int b = s / p.H, h = s - (s / p.H) * p.H;
  const int ch = threadIdx.x % CPR;
  const int g = threadIdx.x / CPR;
  const bool is_q = blk < p.n_qblk;
  const __nv_bfloat16* base;
  long long st;
  int row0, nrows;
  if (is_q) {
    row0 = blk * 64;
    nrows = min(64, p.Lq - row0);
    base = p.q + b * p.q_sb + h * p.q_sh;
    st = p.q_st;
  } else {
    row0 = p.win_row0 + (blk - p.n_qblk) * 64;
    nrows = 64;
    base = p.k + b * p.k_sb + h * p.k_sh;
    st = p.k_st;
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  uint4 v[RPG];
#pragma unroll
  for (int i = 0; i < RPG; ++i) {
    const int r = g * RPG + i;
    v[i] = (r < nrows) ? __ldcs(reinterpret_cast<const uint4*>(base + (long long)(row0 + r) * st) + ch)
                       : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < RPG; ++i) {
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(w[e] << 16);
      acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[g][ch * 8 + e] = acc[e];
  __syncthreads();
  const float inv = 1.f / (float)nrows;
  for (int c = threadIdx.x; c < D; c += 128) {
    float sum = 0.f;
#pragma unroll
    for (int gg = 0; gg < GROUPS; ++gg) sum += part[gg][c];
    float* dst = is_q ? p.qbar + ((size_t)s * p.n_qblk + blk) * D
                      : p.kbar + ((size_t)s * p.n_win + (blk - p.n_qblk)) * D;
    dst[c] = sum * inv;
  }
}

struct SelParams {
  const float* qbar;
  const float* kbar;
  int BH, n_qblk, n_win, topk;
  int* out_idx;
  float* out_scores;
};

// 8 warps per CTA, one warp per (s, query block); scores staged in shared memory.
template <int D>
__global__ void __launch_bounds__(256) select_kernel(const SelParams p) {
  extern __shared__ float sc_all[];  // [8][n_win]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * 8 + warp;
  if (task >= (long long)p.BH * p.n_qblk) return;
  const int s = (int)(task / p.n_qblk);
  const int j = (int)(task - (long long)s * p.n_qblk);
  float* sc = sc_all + warp * p.n_win;
  constexpr int PER = D / 32;
  float qv[PER];
  const float* qrow = p.qbar + ((size_t)s * p.n_qblk + j) * D;
#pragma unroll
  for (int e = 0; e < PER; ++e) qv[e] = qrow[lane * PER + e];
  const float* kb = p.kbar + (size_t)s * p.n_win * D;
  for (int w = 0; w < p.n_win; ++w) {
    const float* kr = kb + (size_t)w * D + lane * PER;
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) part = fmaf(qv[e], kr[e], part);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, o);
    if (lane == 0) {
      sc[w] = (part != part) ? -INFINITY : part;  // NaN ranks last
    }
  }
  __syncwarp();
  if (p.out_scores) {
    float* so = p.out_scores + ((size_t)s * p.n_qblk + j) * p.n_win;
    for (int w = lane; w < p.n_win; w += 32) so[w] = sc[w];
  }
  int* oi = p.out_idx + ((size_t)s * p.n_qblk + j) * p.topk;
  int written = 0;
  for (int w0 = 0; w0 < p.n_win; w0 += 32) {
    const int w = w0 + lane;
    bool keep = false;
    if (w < p.n_win) {
      const float x = sc[w];
      int rank = 0;
      for (int u = 0; u < p.n_win; ++u) {
        const float y = sc[u];
        rank += (y > x) || (y == x && u < w);
      }
      keep = rank < p.topk;
    }
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) oi[written + __popc(bal & ((1u << lane) - 1u))] = w;
    written += __popc(bal);
  }
}

}  // namespace
}  // namespace vkv

using namespace vkv;

extern "C" size_t vkv_block_select_workspace_size(int32_t B, int32_t H, int32_t Lq, int32_t n_win_blk,
                                                  int32_t block, int32_t d) {
  if (B <= 0 || H <= 0 || Lq <= 0 || n_win_blk <= 0 || block <= 0 || d <= 0) return 0;
  const size_t n_qblk = (size_t)(Lq + block - 1) / block;
  const size_t bytes = (size_t)B * H * (n_qblk + (size_t)n_win_blk) * d * sizeof(float);
  return (bytes + 255) & ~(size_t)255;
}

extern "C" vkv_status vkv_block_select(const vkv_select_args* a, vkv_stream_t stream) {
  if (!a) return VKV_ERR_NULL;
  if (a->d != 64 && a->d != 128) return VKV_ERR_UNSUPPORTED;
  if (a->block != 64) return VKV_ERR_UNSUPPORTED;
  if (a->B <= 0 || a->H <= 0 || a->Lq <= 0 || a->Lkv <= 0) return VKV_ERR_SHAPE;
  if (a->n_win_blk < 1 || a->n_win_blk > 1024 || a->topk < 1 || a->topk > a->n_win_blk) return VKV_ERR_SHAPE;
  if (a->window_blk0 < 0 || (long long)(a->window_blk0 + a->n_win_blk) * a->block > a->Lkv) return VKV_ERR_RANGE;
  if (!a->q.ptr || !a->k.ptr || !a->out_idx) return VKV_ERR_NULL;
  if (!tensor_aligned(a->q) || !tensor_aligned(a->k)) return VKV_ERR_ALIGN;
  const size_t need = vkv_block_select_workspace_size(a->B, a->H, a->Lq, a->n_win_blk, a->block, a->d);
  if (!a->workspace || a->workspace_bytes < need) return VKV_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(a->workspace) & 255u) return VKV_ERR_ALIGN;
  if ((long long)a->B * a->H > 65535) return VKV_ERR_UNSUPPORTED;
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int BH = a->B * a->H;
  const int n_qblk = (a->Lq + 63) / 64;
  PoolParams pp;
  pp.q = reinterpret_cast<const __nv_bfloat16*>(a->q.ptr);
  pp.k = reinterpret_cast<const __nv_bfloat16*>(a->k.ptr);
  pp.q_sb = a->q.sb; pp.q_st = a->q.st; pp.q_sh = a->q.sh;
  pp.k_sb = a->k.sb; pp.k_st = a->k.st; pp.k_sh = a->k.sh;
  pp.B = a->B;
  pp.H = a->H;
  pp.d = a->d;
  pp.Lq = a->Lq;
  pp.n_qblk = n_qblk;
  pp.n_win = a->n_win_blk;
  pp.win_row0 = a->window_blk0 * a->block;
  pp.qbar = reinterpret_cast<float*>(a->workspace);
  pp.kbar = pp.qbar + (size_t)BH * n_qblk * a->d;
  dim3 pg(n_qblk + a->n_win_blk, BH);
  if (a->d == 128)
    pool_kernel<128><<<pg, 128, 0, st>>>(pp);
  else
    pool_kernel<64><<<pg, 128, 0, st>>>(pp);
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  SelParams sp;
  sp.qbar = pp.qbar;
  sp.kbar = pp.kbar;
  sp.BH = BH;
  sp.n_qblk = n_qblk;
  sp.n_win = a->n_win_blk;
  sp.topk = a->topk;
  sp.out_idx = a->out_idx;
  sp.out_scores = a->out_scores;
  const long long tasks = (long long)BH * n_qblk;
  const int grid = (int)((tasks + 7) / 8);
  const size_t smem = (size_t)8 * a->n_win_blk * sizeof(float);
  if (a->d == 128)
    select_kernel<128><<<grid, 256, smem, st>>>(sp);
  else
    select_kernel<64><<<grid, 256, smem, st>>>(sp);
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  return VKV_OK;
}

// ---------------------------------------------------------------------------
// vkv_block_select_noalloc: the same selection with library-owned scratch.
//
// Some callers cannot allocate device memory when they call in: a serving
// loop whose device memory was fully planned at start-up and that hands the
// library no allocator, or a host program that drives the library only
// through this C interface and has no way to size, own and free a workspace.
// For them the pooled block vectors live in one file-scope device array of
// fixed size, kNoallocScratchBytes, which every GPU that loads the library
// holds until the process exits.
//
// In host code `g_select_scratch` is only a host-side stand-in for the array;
// its device address is looked up once per device (cudaGetSymbolAddress, with
// that device current) on the first call made on it, and cached.  Every call
// on a device shares the array and leaves the last call's contents behind;
// nothing needs clearing, because every element the select kernel reads is
// written by the pool kernel of the same call.  Calls that overlap on the GPU
// (for example on two streams at once) race on the array.
// ---------------------------------------------------------------------------
namespace vkv {
namespace {

constexpr size_t kNoallocScratchBytes = VKV_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) float g_select_scratch[kNoallocScratchBytes / sizeof(float)];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};

// Device address of the scratch array on the current device; nullptr on failure.
void* noalloc_scratch(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_select_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace vkv

extern "C" vkv_status vkv_block_select_noalloc(const vkv_select_args* a, vkv_stream_t stream) {
  if (!a) return VKV_ERR_NULL;
  if (a->d != 64 && a->d != 128) return VKV_ERR_UNSUPPORTED;
  if (a->block != 64) return VKV_ERR_UNSUPPORTED;
  if (a->B <= 0 || a->H <= 0 || a->Lq <= 0 || a->Lkv <= 0) return VKV_ERR_SHAPE;
  if (a->n_win_blk < 1 || a->n_win_blk > 1024 || a->topk < 1 || a->topk > a->n_win_blk) return VKV_ERR_SHAPE;
  if (a->window_blk0 < 0 || (long long)(a->window_blk0 + a->n_win_blk) * a->block > a->Lkv) return VKV_ERR_RANGE;
  if (!a->q.ptr || !a->k.ptr || !a->out_idx) return VKV_ERR_NULL;
  if (!tensor_aligned(a->q) || !tensor_aligned(a->k)) return VKV_ERR_ALIGN;
  if ((long long)a->B * a->H > 65535) return VKV_ERR_UNSUPPORTED;
  const size_t need = vkv_block_select_workspace_size(a->B, a->H, a->Lq, a->n_win_blk, a->block, a->d);
  if (need > kNoallocScratchBytes) return VKV_ERR_WORKSPACE;  // larger than the fixed scratch array
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  void* scratch = noalloc_scratch(dev);
  if (!scratch) return VKV_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int BH = a->B * a->H;
  const int n_qblk = (a->Lq + 63) / 64;
  PoolParams pp;
  pp.q = reinterpret_cast<const __nv_bfloat16*>(a->q.ptr);
  pp.k = reinterpret_cast<const __nv_bfloat16*>(a->k.ptr);
  pp.q_sb = a->q.sb; pp.q_st = a->q.st; pp.q_sh = a->q.sh;
  pp.k_sb = a->k.sb; pp.k_st = a->k.st; pp.k_sh = a->k.sh;
  pp.B = a->B;
  pp.H = a->H;
  pp.d = a->d;
  pp.Lq = a->Lq;
  pp.n_qblk = n_qblk;
  pp.n_win = a->n_win_blk;
  pp.win_row0 = a->window_blk0 * a->block;
  pp.qbar = reinterpret_cast<float*>(scratch);
  pp.kbar = pp.qbar + (size_t)BH * n_qblk * a->d;
  dim3 pg(n_qblk + a->n_win_blk, BH);
  if (a->d == 128)
    pool_kernel<128><<<pg, 128, 0, st>>>(pp);
  else
    pool_kernel<64><<<pg, 128, 0, st>>>(pp);
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  SelParams sp;
  sp.qbar = pp.qbar;
  sp.kbar = pp.kbar;
  sp.BH = BH;
  sp.n_qblk = n_qblk;
  sp.n_win = a->n_win_blk;
  sp.topk = a->topk;
  sp.out_idx = a->out_idx;
  sp.out_scores = a->out_scores;
  const long long tasks = (long long)BH * n_qblk;
  const int grid = (int)((tasks + 7) / 8);
  const size_t smem = (size_t)8 * a->n_win_blk * sizeof(float);
  if (a->d == 128)
    select_kernel<128><<<grid, 256, smem, st>>>(sp);
  else
    select_kernel<64><<<grid, 256, smem, st>>>(sp);
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  return VKV_OK;
}
