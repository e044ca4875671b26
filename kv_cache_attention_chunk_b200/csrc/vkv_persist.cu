// vkv_persist_update: persistent-memory management (Sparse Forcing summary,
// section 2 component 1 "Structured Memory Decomposition": blocks evicted from
// the local window are candidates, and the top C by coarse score are kept in,
// or replace blocks of, the persistent memory; component 2: one representative
// per block for the coarse score).
//
// Three launches on the caller's stream, the last two as programmatic dependent
// launches (each starts while the one before it drains):
//   pool_kernel          means of the chunk's 64-row query blocks (shared with
//                        block selection) -> workspace;
//   cand_pool_kernel     means of the candidate blocks (current persistent
//                        blocks, then the evicted range) -> workspace, with a
//                        validity flag per candidate;
//   persist_pick_kernel  one CTA per (batch, head): the chunk's mean query from
//                        the block means (weighted by block rows; all threads,
//                        partial sums in shared memory), one score per
//                        candidate (a warp each), rank of each candidate among the valid
//                        ones (higher score first, then the lower block id),
//                        the C best written in ascending block order.
// Candidate counts are small (C + evicted <= 2048), so ranking by counting is
// both exact and cheap.
#include <cstring>

#include "vkv_internal.h"
#include "vkv_pool.cuh"
#include "vkv_ptx.cuh"

namespace vkv {
namespace {

constexpr int kMaxCand = 2048;

struct CandParams {
  const __nv_bfloat16* k;
  long long k_sb, k_st, k_sh;
  const int* persist_idx;  // [BH][C]
  int H, C, n_evict, evict_blk0, n_blocks;
  float* kbar;             // [BH][C + n_evict][d]
  unsigned char* valid;    // [BH][C + n_evict]
  int* err;
};

// grid: x = candidate, y = b*H + h; 256 threads: thread (g, c) sums rows
// g*RPG .. g*RPG + RPG - 1 of 16-byte column c, row groups combined in smem.
template <int D>
__global__ void __launch_bounds__(256) cand_pool_kernel(const CandParams p) {
  constexpr int CPR = D / 8;
  constexpr int GROUPS = 256 / CPR;
  constexpr int RPG = 64 / GROUPS;
  __shared__ float part[GROUPS][D];
  const int i = blockIdx.x;
  const int s = blockIdx.y;
  const int n_cand = p.C + p.n_evict;
  int blk;
  bool ok;
  if (i < p.C) {
    blk = __ldg(p.persist_idx + (size_t)s * p.C + i);
    ok = blk >= 0 && blk < p.n_blocks && (blk < p.evict_blk0 || blk >= p.evict_blk0 + p.n_evict);
    if (!ok && threadIdx.x == 0 && p.err) atomicCAS(p.err, 0, VKV_DEVERR_BAD_INDEX);
  } else {
    blk = p.evict_blk0 + (i - p.C);
    ok = true;
  }
  if (threadIdx.x == 0) p.valid[(size_t)s * n_cand + i] = ok ? 1 : 0;
  if (!ok) {
    griddep_wait();
    return;
  }
  const int b = s / p.H, h = s - (s / p.H) * p.H;
  const int c = threadIdx.x % CPR, g = threadIdx.x / CPR;
  const __nv_bfloat16* base = p.k + b * p.k_sb + h * p.k_sh + (long long)blk * 64 * p.k_st;
  uint4 v[RPG];
#pragma unroll
  for (int r = 0; r < RPG; ++r) v[r] = __ldcs(reinterpret_cast<const uint4*>(base + (long long)(g * RPG + r) * p.k_st) + c);
  // the pick kernel may be scheduled now; it waits for this grid's completion
  griddep_launch_dependents();
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int r = 0; r < RPG; ++r) {
    const uint32_t w[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(w[e] << 16);
      acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[g][c * 8 + e] = acc[e];
  __syncthreads();
  float* dst = p.kbar + ((size_t)s * n_cand + i) * D;
  for (int x = threadIdx.x; x < D; x += 256) {
    float sum = 0.f;
#pragma unroll
    for (int gg = 0; gg < GROUPS; ++gg) sum += part[gg][x];
    dst[x] = sum * (1.f / 64.f);
  }
  // this grid reads nothing the query pooling writes and may run beside it; it ends
  // only after that grid has, so the pick kernel's wait on this grid covers both
  griddep_wait();
}

struct PickParams {
  const float* qbar;            // [BH][n_qblk][d]
  const float* kbar;            // [BH][n_cand][d]
  const unsigned char* valid;   // [BH][n_cand]
  const int* persist_idx;       // [BH][C]
  int C, n_evict, evict_blk0, n_qblk, Lq;
  int* out_idx;                 // [BH][C]
  float* out_scores;            // [BH][n_cand] or null
};

// grid: x = b*H + h; 256 threads.
template <int D>
__global__ void __launch_bounds__(256) persist_pick_kernel(const PickParams p) {
  __shared__ float qm[D];
  __shared__ float sc[kMaxCand];
  __shared__ int ids[kMaxCand];
  __shared__ unsigned char ok[kMaxCand];
  __shared__ unsigned char keep[kMaxCand];
  constexpr int C4 = D / 4;          // 16-byte column chunks of a row
  constexpr int G = 256 / C4;        // row groups
  __shared__ float part[G][D];
  const int s = blockIdx.x;
  const int n_cand = p.C + p.n_evict;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NW = 256 / 32;   // warps
  constexpr int PB = 8;          // candidates a warp holds in registers at once
  constexpr int PL = D / 32;     // columns per lane
  griddep_wait();  // both pooling grids before this one on the stream have completed
  // candidate ids and validity into shared memory (independent loads, all at once)
  for (int i = threadIdx.x; i < n_cand; i += 256) {
    ids[i] = i < p.C ? __ldg(p.persist_idx + (size_t)s * p.C + i) : p.evict_blk0 + (i - p.C);
    ok[i] = p.valid[(size_t)s * n_cand + i];
  }
  // the block means of this warp's first PB candidates (i = warp + NW * b), loaded
  // now so that their latency overlaps the mean-query reduction below
  float kreg[PB][PL];
#pragma unroll
  for (int b = 0; b < PB; ++b) {
    const int i = warp + NW * b;
    const float* kr = p.kbar + ((size_t)s * n_cand + (i < n_cand ? i : 0)) * D;
#pragma unroll
    for (int e = 0; e < PL; ++e) kreg[b][e] = (i < n_cand) ? __ldg(kr + lane + 32 * e) : 0.f;
  }
  // mean query of the chunk: block means weighted by their rows (the last block may
  // be short).  Thread (g, c) sums chunk c of query blocks g, g + G, ... (independent
  // loads, several in flight), then the G partial sums are added in shared memory.
  {
    const int c = threadIdx.x % C4, g = threadIdx.x / C4;
    const float4* qb = reinterpret_cast<const float4*>(p.qbar + (size_t)s * p.n_qblk * D) + c;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int j = g; j < p.n_qblk; j += G) {
      const float w = (float)min(64, p.Lq - j * 64);
      const float4 v = __ldg(qb + (size_t)j * C4);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    part[g][4 * c + 0] = acc.x;
    part[g][4 * c + 1] = acc.y;
    part[g][4 * c + 2] = acc.z;
    part[g][4 * c + 3] = acc.w;
  }
  __syncthreads();
  for (int x = threadIdx.x; x < D; x += blockDim.x) {
    float acc = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) acc += part[g][x];
    qm[x] = acc / (float)p.Lq;
  }
  __syncthreads();
  // one warp per candidate: lane l takes columns l, l + 32, ... of the block mean
  // (the first PB candidates of each warp from the registers loaded above)
  for (int i = warp, b = 0; i < n_cand; i += NW, ++b) {
    const bool valid = ok[i] != 0;
    float v = -INFINITY;
    if (valid) {
      float a = 0.f;
      if (b < PB) {
#pragma unroll
        for (int bb = 0; bb < PB; ++bb)
          if (bb == b) {
#pragma unroll
            for (int e = 0; e < PL; ++e) a = fmaf(qm[lane + 32 * e], kreg[bb][e], a);
          }
      } else {
        const float* kr = p.kbar + ((size_t)s * n_cand + i) * D;
#pragma unroll
        for (int e = 0; e < PL; ++e) a = fmaf(qm[lane + 32 * e], __ldg(kr + lane + 32 * e), a);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
      v = (a != a) ? -INFINITY : (a == 0.f ? 0.f : a);  // NaN ranks last; -0 ties with +0
    }
    if (lane == 0) {
      sc[i] = v;
      if (p.out_scores) p.out_scores[(size_t)s * n_cand + i] = valid ? v : -INFINITY;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_cand; i += blockDim.x) {
    int rank = 0;
    const float si = sc[i];
    const int di = ids[i];
    for (int j = 0; j < n_cand; ++j)
      rank += (ok[j] && (sc[j] > si || (sc[j] == si && ids[j] < di))) ? 1 : 0;
    keep[i] = (ok[i] && rank < p.C) ? 1 : 0;
  }
  __syncthreads();
  int* out = p.out_idx + (size_t)s * p.C;
  for (int i = threadIdx.x; i < n_cand; i += blockDim.x) {
    if (!keep[i]) continue;
    int pos = 0;
    for (int j = 0; j < n_cand; ++j) pos += (keep[j] && ids[j] < ids[i]) ? 1 : 0;
    out[pos] = ids[i];
  }
  // fewer than C valid candidates (only after an invalid persistent id): pad with -1
  __syncthreads();
  if (threadIdx.x == 0) {
    int kept = 0;
    for (int i = 0; i < n_cand; ++i) kept += keep[i];
    for (int x = kept; x < p.C; ++x) out[x] = -1;
  }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Programmatic dependent launch of a 256-thread kernel with one parameter struct:
// the grid may start while the one before it on the stream is still running, and
// orders itself with griddep_wait.
template <class P>
bool launch_dependent(const void* fn, dim3 grid, cudaStream_t st, P* params) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[1] = {params};
  return cudaLaunchKernelExC(&cfg, fn, args) == cudaSuccess;
}

}  // namespace
}  // namespace vkv

using namespace vkv;

extern "C" size_t vkv_persist_update_workspace_size(int32_t B, int32_t H, int32_t Lq, int32_t n_persist,
                                                    int32_t n_evict, int32_t block, int32_t d) {
  if (B <= 0 || H <= 0 || Lq <= 0 || n_persist <= 0 || n_evict < 0 || block <= 0 || d <= 0) return 0;
  const size_t BH = (size_t)B * H;
  const size_t n_qblk = (size_t)(Lq + block - 1) / block;
  const size_t n_cand = (size_t)n_persist + n_evict;
  return align256(BH * n_qblk * d * sizeof(float)) + align256(BH * n_cand * d * sizeof(float)) +
         align256(BH * n_cand);
}

extern "C" vkv_status vkv_persist_update(const vkv_persist_args* a, vkv_stream_t stream) {
  if (!a) return VKV_ERR_NULL;
  if (a->d != 64 && a->d != 128) return VKV_ERR_UNSUPPORTED;
  if (a->block != 64) return VKV_ERR_UNSUPPORTED;
  if (a->B <= 0 || a->H <= 0 || a->Lq <= 0 || a->Lkv <= 0) return VKV_ERR_SHAPE;
  if (a->n_persist < 1 || a->n_persist > 1024 || a->n_evict < 0 || a->n_evict > 1024) return VKV_ERR_SHAPE;
  if (a->evict_blk0 < 0 || (long long)(a->evict_blk0 + a->n_evict) * a->block > a->Lkv) return VKV_ERR_RANGE;
  if (!a->q.ptr || !a->k.ptr || !a->persist_idx || !a->out_idx) return VKV_ERR_NULL;
  if (!tensor_aligned(a->q) || !tensor_aligned(a->k)) return VKV_ERR_ALIGN;
  if ((long long)a->B * a->H > 65535) return VKV_ERR_UNSUPPORTED;
  const size_t need = vkv_persist_update_workspace_size(a->B, a->H, a->Lq, a->n_persist, a->n_evict, a->block, a->d);
  if (!a->workspace || a->workspace_bytes < need) return VKV_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(a->workspace) & 255u) return VKV_ERR_ALIGN;
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int BH = a->B * a->H;
  const int n_qblk = (a->Lq + 63) / 64;
  const int n_cand = a->n_persist + a->n_evict;
  uint8_t* ws = reinterpret_cast<uint8_t*>(a->workspace);
  float* qbar = reinterpret_cast<float*>(ws);
  float* kbar = reinterpret_cast<float*>(ws + align256((size_t)BH * n_qblk * a->d * sizeof(float)));
  unsigned char* valid = reinterpret_cast<unsigned char*>(kbar) + align256((size_t)BH * n_cand * a->d * sizeof(float));
  // 1. query block means
  PoolParams pp;
  std::memset(&pp, 0, sizeof(pp));
  pp.q = reinterpret_cast<const __nv_bfloat16*>(a->q.ptr);
  pp.q_sb = a->q.sb; pp.q_st = a->q.st; pp.q_sh = a->q.sh;
  pp.B = a->B;
  pp.H = a->H;
  pp.d = a->d;
  pp.Lq = a->Lq;
  pp.n_qblk = n_qblk;
  pp.n_win = 0;
  pp.qbar = qbar;
  const int ph = a->d == 128 ? pool_heads<128>() : pool_heads<64>();
  const dim3 pg(n_qblk, a->B * ((a->H + ph - 1) / ph));
  if (a->d == 128)
    pool_kernel<128><<<pg, 256, 0, st>>>(pp);
  else
    pool_kernel<64><<<pg, 256, 0, st>>>(pp);
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  // 2. candidate block means
  CandParams cp;
  cp.k = reinterpret_cast<const __nv_bfloat16*>(a->k.ptr);
  cp.k_sb = a->k.sb; cp.k_st = a->k.st; cp.k_sh = a->k.sh;
  cp.persist_idx = a->persist_idx;
  cp.H = a->H;
  cp.C = a->n_persist;
  cp.n_evict = a->n_evict;
  cp.evict_blk0 = a->evict_blk0;
  cp.n_blocks = a->Lkv / 64;
  cp.kbar = kbar;
  cp.valid = valid;
  cp.err = a->err_word;
  if (!launch_dependent(a->d == 128 ? (const void*)cand_pool_kernel<128> : (const void*)cand_pool_kernel<64>,
                        dim3(n_cand, BH), st, &cp))
    return VKV_ERR_CUDA;
  // 3. scores and the top C
  PickParams kp;
  kp.qbar = qbar;
  kp.kbar = kbar;
  kp.valid = valid;
  kp.persist_idx = a->persist_idx;
  kp.C = a->n_persist;
  kp.n_evict = a->n_evict;
  kp.evict_blk0 = a->evict_blk0;
  kp.n_qblk = n_qblk;
  kp.Lq = a->Lq;
  kp.out_idx = a->out_idx;
  kp.out_scores = a->out_scores;
  if (!launch_dependent(a->d == 128 ? (const void*)persist_pick_kernel<128> : (const void*)persist_pick_kernel<64>,
                        dim3(BH), st, &kp))
    return VKV_ERR_CUDA;
  return VKV_OK;
}
