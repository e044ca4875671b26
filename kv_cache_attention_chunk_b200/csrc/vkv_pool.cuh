// Block pooling shared by block selection and persistent-memory management:
// the representative of a 64-row block is the fp32 mean of its rows (Sparse
// Forcing summary, section 2 component 2 "Blockified Compression").
#pragma once

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

// Heads per pooling CTA: a contiguous 1024-byte slice of each row (4 heads at
// d = 128, 8 at d = 64), 16 rows per thread in flight.
#ifndef VKV_POOL_SLICE
#define VKV_POOL_SLICE 1024
#endif
template <int D>
__host__ __device__ constexpr int pool_heads() { return VKV_POOL_SLICE / (2 * D) > 0 ? VKV_POOL_SLICE / (2 * D) : 1; }

// grid: x = first block index (the CTA then steps over blocks by gridDim.x, so a
// grid narrower than the block count leaves room on every SM for a dependent
// kernel), y = b * ceil(H / kPoolHeads) + head group; 256 threads.  Thread (g, c):
// column c = (head, 16-byte chunk) of the head group's slice, rows g*RPG ..
// g*RPG + RPG - 1 of the 64-row block; the row groups are combined in shared memory.
#ifndef VKV_POOL_MINB
#define VKV_POOL_MINB 2
#endif
template <int D>
__global__ void __launch_bounds__(256, VKV_POOL_MINB) pool_kernel(const PoolParams p) {
  constexpr int kPoolHeads = pool_heads<D>();
  constexpr int CPR = D / 8;                  // 16-byte chunks per head row
  constexpr int COLS = kPoolHeads * CPR;      // columns of the slice
  constexpr int GROUPS = 256 / COLS;          // row groups
  constexpr int RPG = 64 / GROUPS;            // rows per group
  __shared__ float part[GROUPS][COLS * 8];
  const int n_hg = (p.H + kPoolHeads - 1) / kPoolHeads;
  const int b = blockIdx.y / n_hg;
  const int h0 = (blockIdx.y - b * n_hg) * kPoolHeads;
  const int nh = min(kPoolHeads, p.H - h0);
  const int c = threadIdx.x % COLS;
  const int g = threadIdx.x / COLS;
  const int hc = c / CPR, ch = c % CPR;
  const bool col_ok = hc < nh;
  // the kernel behind this one (block selection) may be scheduled now: it waits
  // for this grid's completion before it reads a pooled vector
  griddep_launch_dependents();
  for (int blk = blockIdx.x; blk < p.n_qblk + p.n_win; blk += gridDim.x) {
    const bool is_q = blk < p.n_qblk;
    const __nv_bfloat16* base;
    long long st;
    int row0, nrows;
    if (is_q) {
      row0 = blk * 64;
      nrows = min(64, p.Lq - row0);
      base = p.q + b * p.q_sb + (h0 + hc) * p.q_sh;
      st = p.q_st;
    } else {
      row0 = p.win_row0 + (blk - p.n_qblk) * 64;
      nrows = 64;
      base = p.k + b * p.k_sb + (h0 + hc) * p.k_sh;
      st = p.k_st;
    }
    uint4 v[RPG];
#pragma unroll
    for (int i = 0; i < RPG; ++i) {
      const int r = g * RPG + i;
      v[i] = (col_ok && r < nrows)
                 ? __ldcs(reinterpret_cast<const uint4*>(base + (long long)(row0 + r) * st) + ch)
                 : make_uint4(0, 0, 0, 0);
    }
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int i = 0; i < RPG; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += __uint_as_float(w[e] << 16);
        acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
    __syncthreads();  // the previous block's sums have been read
#pragma unroll
    for (int e = 0; e < 8; ++e) part[g][c * 8 + e] = acc[e];
    __syncthreads();
    const float inv = 1.f / (float)nrows;
    for (int x = threadIdx.x; x < COLS * 8; x += 256) {
      const int hx = x / D, cx = x % D;
      if (hx >= nh) continue;
      float sum = 0.f;
#pragma unroll
      for (int gg = 0; gg < GROUPS; ++gg) sum += part[gg][x];
      const int s = b * p.H + h0 + hx;
      float* dst = is_q ? p.qbar + ((size_t)s * p.n_qblk + blk) * D
                        : p.kbar + ((size_t)s * p.n_win + (blk - p.n_qblk)) * D;
      dst[cx] = sum * inv;
    }
  }
}

}  // namespace
}  // namespace vkv
