// vkv_persist_update: persistent-memory management (Sparse Forcing summary,
// section 2 component 1 "Structured Memory Decomposition": blocks evicted from
// the local window are candidates, and the top C by coarse score are kept in,
// or replace blocks of, the persistent memory; component 2: one representative
// per block for the coarse score).
//
// One launch: a thread-block cluster of kPersistSplit CTAs per (batch, head).
//   1. every CTA sums its slice of the chunk's query rows (16-byte column chunks,
//      16 rows per thread in flight) into its shared memory, and each of its
//      warps takes one of the CTA's candidate blocks (the current persistent
//      blocks, then the evicted range; candidates rank, rank + kPersistSplit,
//      ...): the block's mean, lanes adding their row subsets by shuffles, to
//      the workspace;
//   2. after a cluster barrier every CTA adds the CTAs' query sums from their
//      shared memory (distributed shared memory, in rank order: every CTA gets
//      the same mean query) and scores its own candidates (the warp that
//      pooled a block scores it), writing the scores into CTA 0's shared memory;
//   3. after a second cluster barrier CTA 0 ranks every candidate among the
//      valid ones (higher score first, then the lower block id) by counting and
//      writes the C best in ascending block order.
// Candidate counts are small (C + evicted <= 2048), so ranking by counting is
// both exact and cheap.
#include <cstring>

#include "vkv_internal.h"
#include "vkv_ptx.cuh"

namespace vkv {
namespace {

// Thread-block clusters: the CTA's rank, the cluster barrier, and the shared memory
// of another CTA of the cluster (distributed shared memory).
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of every CTA of the cluster: memory operations before it (shared
// and global) are visible to all the cluster's threads after it.  All threads of
// the cluster must execute it the same number of times.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Stores v into CTA `rank`'s shared memory, at the offset of `local` in this CTA's.
__device__ __forceinline__ void dsmem_st_f32(float* local, uint32_t rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}

// A float of CTA `rank`'s shared memory, at the offset of `local` in this CTA's.
__device__ __forceinline__ float dsmem_ld_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

constexpr int kMaxCand = 2048;
constexpr int kPersistSplit = 8;  // CTAs per (batch, head): one cluster

struct PersistParams {
  const __nv_bfloat16* q;
  long long q_sb, q_st, q_sh;
  const __nv_bfloat16* k;
  long long k_sb, k_st, k_sh;
  const int* persist_idx;  // [BH][C]
  int H, Lq, C, n_evict, evict_blk0, n_blocks;
  float* kbar;             // workspace [BH][C + n_evict][d]: the candidates' block means
  int* out_idx;            // [BH][C]
  float* out_scores;       // [BH][C + n_evict] or null
  int* err;
};

// Candidate i of sequence s: its block id, and whether it may be ranked (a
// persistent id inside the cache and outside the evicted range).
__device__ __forceinline__ int cand_block(const PersistParams& p, int s, int i, bool& ok) {
  if (i < p.C) {
    const int blk = __ldg(p.persist_idx + (size_t)s * p.C + i);
    ok = blk >= 0 && blk < p.n_blocks && (blk < p.evict_blk0 || blk >= p.evict_blk0 + p.n_evict);
    return blk;
  }
  ok = true;
  return p.evict_blk0 + (i - p.C);
}

__device__ __forceinline__ void add_bf16x8(float* acc, const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    acc[2 * e] += __uint_as_float(w[e] << 16);
    acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

// grid: x = kPersistSplit (one cluster), y = b*H + h; 256 threads.
template <int D>
__global__ void __cluster_dims__(kPersistSplit, 1, 1) __launch_bounds__(256)
    persist_update_kernel(const PersistParams p) {
  constexpr int CPR = D / 8;     // 16-byte chunks per row
  constexpr int G = 256 / CPR;   // row groups of the query sum
  constexpr int RS = 32 / CPR;   // row subsets of a warp pooling one block
  constexpr int PL = D / 32;     // columns per lane when a warp scores a block
  constexpr int NW = 256 / 32;
  constexpr int QU = 16;         // query rows per thread in flight
  __shared__ float part[G][D];
  __shared__ float qpart[D];     // this CTA's sum of its query rows (read by every CTA)
  __shared__ float qm[D];
  __shared__ float sc[kMaxCand];  // CTA 0: every candidate's score
  __shared__ int ids[kMaxCand];   // CTA 0: block id, then (INT_MAX unless kept) for the output order
  __shared__ unsigned long long rk[kMaxCand];  // CTA 0: ranking key (0 for an invalid candidate)
  __shared__ int n_valid;
  const uint32_t rank = cluster_ctarank();
  const int s = blockIdx.y;
  const int b = s / p.H, h = s - (s / p.H) * p.H;
  const int n_cand = p.C + p.n_evict;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 1a. the sum of this CTA's slice of the query rows; thread (g, c): chunk c of
  //     rows r0 + g, r0 + g + G, ...
  {
    const int c = threadIdx.x % CPR, g = threadIdx.x / CPR;
    const int R = (p.Lq + kPersistSplit - 1) / kPersistSplit;
    const int r0 = (int)rank * R, r1 = min(p.Lq, r0 + R);
    const __nv_bfloat16* base = p.q + b * p.q_sb + h * p.q_sh;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int row0 = r0 + g; row0 < r1; row0 += QU * G) {
      uint4 v[QU];
#pragma unroll
      for (int u = 0; u < QU; ++u) {
        const int row = row0 + u * G;
        v[u] = row < r1 ? __ldcs(reinterpret_cast<const uint4*>(base + (long long)row * p.q_st) + c)
                        : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < QU; ++u) add_bf16x8(acc, v[u]);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[g][c * 8 + e] = acc[e];
  }
  // 1b. warp w pools candidates rank + kPersistSplit * (w + NW * t): lane (sub, c) sums
  //     chunk c of rows sub, sub + RS, ..., then the row subsets are added by shuffles
  const __nv_bfloat16* kbase = p.k + b * p.k_sb + h * p.k_sh;
  {
    const int c = lane % CPR, sub = lane / CPR;
    for (int i = (int)rank + kPersistSplit * warp; i < n_cand; i += kPersistSplit * NW) {
      bool v_ok = false;
      const int blk = cand_block(p, s, i, v_ok);
      if (!v_ok) continue;
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int r0 = 0; r0 < 64 / RS; r0 += 16) {
        uint4 v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u)
          v[u] = __ldcs(reinterpret_cast<const uint4*>(kbase + ((long long)blk * 64 + sub + RS * (r0 + u)) * p.k_st) + c);
#pragma unroll
        for (int u = 0; u < 16; ++u) add_bf16x8(acc, v[u]);
      }
#pragma unroll
      for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xFFFFFFFFu, acc[e], o);
      if (sub == 0) {
        float4* dst = reinterpret_cast<float4*>(p.kbar + ((size_t)s * n_cand + i) * D + c * 8);
        dst[0] = make_float4(acc[0] * (1.f / 64.f), acc[1] * (1.f / 64.f), acc[2] * (1.f / 64.f), acc[3] * (1.f / 64.f));
        dst[1] = make_float4(acc[4] * (1.f / 64.f), acc[5] * (1.f / 64.f), acc[6] * (1.f / 64.f), acc[7] * (1.f / 64.f));
      }
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < D; x += 256) {
    float t = 0.f;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) t += part[gg][x];
    qpart[x] = t;
  }
  // 2. the mean query from every CTA's sum (the same order in every CTA), then the
  //    scores of this CTA's candidates into CTA 0's shared memory
  cluster_sync();
  for (int x = threadIdx.x; x < D; x += 256) {
    float v[kPersistSplit];
#pragma unroll
    for (uint32_t r = 0; r < kPersistSplit; ++r) v[r] = dsmem_ld_f32(&qpart[x], r);
    float t = 0.f;
#pragma unroll
    for (uint32_t r = 0; r < kPersistSplit; ++r) t += v[r];
    qm[x] = t / (float)p.Lq;
  }
  __syncthreads();
  for (int i = (int)rank + kPersistSplit * warp; i < n_cand; i += kPersistSplit * NW) {
    bool v_ok = false;
    cand_block(p, s, i, v_ok);
    float v = -INFINITY;
    if (v_ok) {
      // the block mean this warp wrote in step 1 (ordered by the barriers since)
      const float* kr = p.kbar + ((size_t)s * n_cand + i) * D;
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < PL; ++e) a = fmaf(qm[lane + 32 * e], __ldcg(kr + lane + 32 * e), a);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
      v = (a != a) ? -INFINITY : (a == 0.f ? 0.f : a);  // NaN ranks last; -0 ties with +0
    }
    if (lane == 0) {
      dsmem_st_f32(&sc[i], 0, v);
      if (p.out_scores) p.out_scores[(size_t)s * n_cand + i] = v;
    }
  }
  cluster_sync();  // every score is in CTA 0; no CTA reads another's memory after this
  if (rank != 0) return;
  // 3. rank by counting.  A valid candidate's key is its score's order-preserving
  //    image above the complement of its block id (higher score first, then the
  //    lower id); an invalid one's key is 0, below every valid key.
  if (threadIdx.x == 0) n_valid = 0;
  __syncthreads();
  int my_valid = 0;
  int my_id[kMaxCand / 256];
  unsigned long long my_key[kMaxCand / 256];
#pragma unroll
  for (int t = 0; t < kMaxCand / 256; ++t) {
    const int i = threadIdx.x + 256 * t;
    my_id[t] = 0;
    my_key[t] = 0ull;
    if (i < n_cand) {
      bool v = false;
      my_id[t] = cand_block(p, s, i, v);
      if (!v && p.err) atomicCAS(p.err, 0, VKV_DEVERR_BAD_INDEX);
      if (v) {
        const uint32_t u = __float_as_uint(sc[i]);
        my_key[t] = ((unsigned long long)(u ^ ((u >> 31) ? 0xFFFFFFFFu : 0x80000000u)) << 32) |
                    (unsigned long long)(0xFFFFFFFFu - (uint32_t)my_id[t]);
        ++my_valid;
      }
      rk[i] = my_key[t];
    }
  }
  if (my_valid) atomicAdd(&n_valid, my_valid);
  __syncthreads();
  // the kept ones' ids (the others INT_MAX) give the ascending output positions
#pragma unroll
  for (int t = 0; t < kMaxCand / 256; ++t) {
    const int i = threadIdx.x + 256 * t;
    if (i >= n_cand) break;
    int r = 0;
#pragma unroll 8
    for (int j = 0; j < n_cand; ++j) r += rk[j] > my_key[t] ? 1 : 0;
    ids[i] = (my_key[t] != 0ull && r < p.C) ? my_id[t] : 0x7FFFFFFF;
  }
  __syncthreads();
  int* out = p.out_idx + (size_t)s * p.C;
#pragma unroll
  for (int t = 0; t < kMaxCand / 256; ++t) {
    const int i = threadIdx.x + 256 * t;
    if (i >= n_cand) break;
    const int id = ids[i];
    if (id == 0x7FFFFFFF) continue;
    int pos = 0;
#pragma unroll 8
    for (int j = 0; j < n_cand; ++j) pos += ids[j] < id ? 1 : 0;
    out[pos] = id;
  }
  // fewer than C valid candidates (only after an invalid persistent id): pad with -1
  for (int x = min(p.C, n_valid) + (int)threadIdx.x; x < p.C; x += 256) out[x] = -1;
}

}  // namespace
}  // namespace vkv

using namespace vkv;

extern "C" size_t vkv_persist_update_workspace_size(int32_t B, int32_t H, int32_t Lq, int32_t n_persist,
                                                    int32_t n_evict, int32_t block, int32_t d) {
  if (B <= 0 || H <= 0 || Lq <= 0 || n_persist <= 0 || n_evict < 0 || block <= 0 || d <= 0) return 0;
  // the candidates' block means
  const size_t bytes = (size_t)B * H * ((size_t)n_persist + n_evict) * d * sizeof(float);
  return (bytes + 255) & ~(size_t)255;
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
  PersistParams pp;
  std::memset(&pp, 0, sizeof(pp));
  pp.q = reinterpret_cast<const __nv_bfloat16*>(a->q.ptr);
  pp.q_sb = a->q.sb; pp.q_st = a->q.st; pp.q_sh = a->q.sh;
  pp.k = reinterpret_cast<const __nv_bfloat16*>(a->k.ptr);
  pp.k_sb = a->k.sb; pp.k_st = a->k.st; pp.k_sh = a->k.sh;
  pp.persist_idx = a->persist_idx;
  pp.H = a->H;
  pp.Lq = a->Lq;
  pp.C = a->n_persist;
  pp.n_evict = a->n_evict;
  pp.evict_blk0 = a->evict_blk0;
  pp.n_blocks = a->Lkv / 64;
  pp.kbar = reinterpret_cast<float*>(a->workspace);
  pp.out_idx = a->out_idx;
  pp.out_scores = a->out_scores;
  pp.err = a->err_word;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(kPersistSplit, (unsigned)(a->B * a->H));
  if (a->d == 128)
    persist_update_kernel<128><<<grid, 256, 0, st>>>(pp);
  else
    persist_update_kernel<64><<<grid, 256, 0, st>>>(pp);
  return cudaGetLastError() == cudaSuccess ? VKV_OK : VKV_ERR_CUDA;
}
