// vkv_block_select: blockified coarse scoring and top-K window-block selection
// (Sparse Forcing summary, section 2 component 2 "Blockified Compression": one
// representative token per block for coarse scoring; component 3 "PBSA":
// top-K blocks of the local window, per query block).
//
// Kernels on the caller's stream:
//   pool_kernel     (unless the caller passes cached window block means) the
//                   fp32 mean of every 64-row window block of K, written to the
//                   caller's workspace.  One CTA of 256 threads per (block,
//                   batch, group of 512/d heads): the group's contiguous slice of
//                   each row is read with 16-byte loads, 16 rows per thread in
//                   flight; row groups are combined in shared memory.  HBM-bound.
//   select_kernel   one CTA per (batch*head, 4 query blocks): pools its query
//                   blocks from Q into shared memory, scores them against the
//                   window block means and keeps the exact top-K by counting
//                   (below).  Launched as a programmatic dependent of the
//                   pooling kernel, so its query pooling overlaps the window
//                   pooling; it reads the window means only after the wait.
//   order_kernel    (optional) the query-block order that groups similar
//                   selections.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "vkv_internal.h"
#include "vkv_pool.cuh"
#include "vkv_ptx.cuh"
#include "vkv_topk.cuh"

namespace vkv {

namespace {

struct SelParams {
  const __nv_bfloat16* q;
  long long q_sb, q_st, q_sh;
  const float* kbar;  // [B*H][n_win][D] window block means
  int H, Lq, n_qblk, n_win, topk;
  int* out_idx;
  float* out_scores;
  int* err;
  int stage;  // the head's window means are copied to shared memory (they fit)
};

constexpr int kSelQ = 4;                    // query blocks per CTA (one warp each for the top-K)
constexpr int kSelStageBytes = 96 * 1024;   // largest staged window (n_win * D * 4 bytes)

// Shared memory of the selection kernel (bytes): the staged window means
// [n_win][D] fp32 (when they fit in kSelStageBytes), the pooled queries
// [kSelQ][D] fp32, the row-group partial sums [G][kSelQ * D] fp32 -- whose space
// later holds the ranking keys [kSelQ][n_win] uint32 --, one 256-bin digit
// histogram per query block, an mbarrier and an abort flag.
template <int D>
constexpr size_t sel_part_bytes() { return (size_t)(256 / (D / 8)) * kSelQ * D * sizeof(float); }
template <int D>
constexpr int sel_row_stride() { return D + 4; }  // floats per staged row: conflict-free column reads
template <int D>
size_t sel_smem_bytes(int n_win, bool stage) {
  return (stage ? (size_t)n_win * sel_row_stride<D>() * sizeof(float) : 0) + (size_t)kSelQ * D * sizeof(float) +
         sel_part_bytes<D>() + (size_t)kSelQ * 256 * sizeof(int) + 16;
}

// grid: x = ceil(n_qblk / kSelQ), y = b*H + h; 256 threads.
//  0. After the window pooling kernel before it (if any) has completed, warp 0
//     starts one bulk copy per window block mean into shared memory (when they
//     fit), into rows padded to d + 4 floats; they land while the query blocks
//     are pooled.
//  1. Pool the CTA's kSelQ query blocks from q: thread (g, c) sums 16-byte column
//     chunk c of rows g, g + G, ... of every block (all loads in flight at
//     once), the row groups are added in shared memory, then divided by the
//     block's row count.
//  2. Thread w scores window block w against the kSelQ pooled queries from its
//     staged row (the padding puts the rows of a quarter-warp in different
//     banks; every row is summed in the same order, so equal block means give
//     equal scores); without staging, a warp reads whole block means from
//     global memory and adds the lanes' partial products by shuffles.  NaN
//     scores rank last and -0 counts as +0, so equal scores tie on the block
//     index.  A score becomes its order-preserving 32-bit integer image (larger
//     score, larger key).
//  3. Warp q selects the top-K of query block q on its own (warp_topk: radix
//     selection of the K-th largest key, then a ballot gives each kept block
//     its output position).
template <int D>
__global__ void __launch_bounds__(256) select_kernel(const SelParams p) {
  constexpr int CPR = D / 8;     // 16-byte chunks per row (bf16)
  constexpr int G = 256 / CPR;   // row groups
  constexpr int RPT = 64 / G;    // rows per thread and block
  constexpr int CH = D / 4;      // 16-byte chunks per block mean (fp32)
  extern __shared__ __align__(16) uint8_t sel_sm[];
  constexpr int RS = sel_row_stride<D>();
  const size_t stage_bytes = p.stage ? (size_t)p.n_win * RS * sizeof(float) : 0;
  float* kbs = reinterpret_cast<float*>(sel_sm);                                      // [n_win][D + 4] (staged)
  float* qs = reinterpret_cast<float*>(sel_sm + stage_bytes);                         // [kSelQ][D]
  float* part = qs + kSelQ * D;                                                       // [G][kSelQ * D]
  uint32_t* keys = reinterpret_cast<uint32_t*>(part);                                 // [kSelQ][n_win] (after part)
  int* hist = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(part) + sel_part_bytes<D>());  // [kSelQ][256]
  uint64_t* bar = reinterpret_cast<uint64_t*>(hist + kSelQ * 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 1);
  const int s = blockIdx.y;
  const int b = s / p.H, h = s - (s / p.H) * p.H;
  const int j0 = blockIdx.x * kSelQ;
  const int nq = min(kSelQ, p.n_qblk - j0);
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const uint32_t b_kb = smem_u32(bar);
  const float* kb_head = p.kbar + (size_t)s * p.n_win * D;
  if (tid == 0) {
    mbar_init(b_kb, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();  // the window pooling kernel before this one (if any) has completed
  if (p.stage && warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(b_kb, (uint32_t)(p.n_win * D * sizeof(float)));
    __syncwarp();
    for (int w = lane; w < p.n_win; w += 32)
      bulk_load(smem_u32(kbs + (size_t)w * RS), kb_head + (size_t)w * D, (uint32_t)(D * sizeof(float)), b_kb);
  }
  // 1. pooled query blocks
  {
    const int c = tid % CPR, g = tid / CPR;
    const __nv_bfloat16* base = p.q + b * p.q_sb + h * p.q_sh;
    uint4 v[kSelQ][RPT];
#pragma unroll
    for (int q = 0; q < kSelQ; ++q)
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int row = (j0 + q) * 64 + g + G * i;
        v[q][i] = (q < nq && row < p.Lq)
                      ? __ldcs(reinterpret_cast<const uint4*>(base + (long long)row * p.q_st) + c)
                      : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
    for (int q = 0; q < kSelQ; ++q) {
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const uint32_t w[4] = {v[q][i].x, v[q][i].y, v[q][i].z, v[q][i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += __uint_as_float(w[e] << 16);
          acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
        }
      }
      float4* dst = reinterpret_cast<float4*>(part + (size_t)g * kSelQ * D + q * D + c * 8);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
  __syncthreads();
  for (int x = tid; x < kSelQ * D; x += 256) {
    const int q = x / D;
    float sum = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) sum += part[(size_t)g * kSelQ * D + x];
    const int nrows = q < nq ? min(64, p.Lq - (j0 + q) * 64) : 1;
    qs[x] = sum * (1.f / (float)nrows);
  }
  __syncthreads();  // part is dead from here on: its space holds the keys
  // 2. scores
  if (p.stage) {
    if (!mbar_wait(b_kb, 0, abort_flag, p.err)) {
      // the copy did not arrive in time: let it land before the CTA exits
      if (tid == 0) mbar_wait_drain(b_kb, 0);
      return;
    }
    for (int w = tid; w < p.n_win; w += 256) {
      const float4* kr = reinterpret_cast<const float4*>(kbs + (size_t)w * RS);
      uint64_t acc[kSelQ][2];  // per query block: chains (x, y) and (z, w), two per f32x2 multiply-add
#pragma unroll
      for (int q = 0; q < kSelQ; ++q) acc[q][0] = acc[q][1] = 0ull;
#pragma unroll 8
      for (int cc = 0; cc < CH; ++cc) {
        const float4 kv = kr[cc];
        const uint64_t k01 = pack2f(kv.x, kv.y), k23 = pack2f(kv.z, kv.w);
#pragma unroll
        for (int q = 0; q < kSelQ; ++q) {
          const float4 qv = reinterpret_cast<const float4*>(qs + q * D)[cc];
          acc[q][0] = fma2f(pack2f(qv.x, qv.y), k01, acc[q][0]);
          acc[q][1] = fma2f(pack2f(qv.z, qv.w), k23, acc[q][1]);
        }
      }
#pragma unroll
      for (int q = 0; q < kSelQ; ++q) {
        float a0, a1, a2, a3;
        unpack2f(acc[q][0], a0, a1);
        unpack2f(acc[q][1], a2, a3);
        const float v = rank_score((a0 + a1) + (a2 + a3));
        if (q < nq && p.out_scores) p.out_scores[((size_t)s * p.n_qblk + j0 + q) * p.n_win + w] = v;
        keys[q * p.n_win + w] = score_key(v);
      }
    }
  } else {
    // a warp reads whole block means (lane l: 16-byte chunk l % CH of row w0 + l / CH),
    // six rows of each lane in flight; the lanes' partial products are added by shuffles
    constexpr int RPW = 32 / CH;
    constexpr int kRows = 6;
    const int c = lane % CH, rsub = lane / CH;
    for (int w0 = warp * RPW; w0 < p.n_win; w0 += 8 * RPW * kRows) {
      float4 kv[kRows];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int w = w0 + i * 8 * RPW + rsub;
        kv[i] = w < p.n_win ? __ldg(reinterpret_cast<const float4*>(kb_head + (size_t)w * D) + c)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int w = w0 + i * 8 * RPW + rsub;
        float sc[kSelQ];
#pragma unroll
        for (int q = 0; q < kSelQ; ++q) {
          const float4 qv = reinterpret_cast<const float4*>(qs + q * D)[c];
          sc[q] = fmaf(qv.x, kv[i].x, fmaf(qv.y, kv[i].y, fmaf(qv.z, kv[i].z, qv.w * kv[i].w)));
        }
#pragma unroll
        for (int o = CH / 2; o > 0; o >>= 1)
#pragma unroll
          for (int q = 0; q < kSelQ; ++q) sc[q] += __shfl_xor_sync(0xFFFFFFFFu, sc[q], o);
        if (c < kSelQ && w < p.n_win) {
          float v = sc[0];
#pragma unroll
          for (int q = 1; q < kSelQ; ++q) v = (c == q) ? sc[q] : v;
          v = rank_score(v);
          if (c < nq && p.out_scores) p.out_scores[((size_t)s * p.n_qblk + j0 + c) * p.n_win + w] = v;
          keys[c * p.n_win + w] = score_key(v);
        }
      }
    }
  }
  __syncthreads();
  // 3. warp q: top-K of query block q
  if (warp >= nq) return;
  warp_topk(keys + warp * p.n_win, p.n_win, p.topk, hist + warp * 256,
            p.out_idx + ((size_t)s * p.n_qblk + j0 + warp) * p.topk, nullptr);
}

// Query-block order that groups blocks with similar selections (a work-grouping
// aid for the block-sparse attention, not part of the selection itself).
// Signature of query block j: its first kOrderIds selected ids (ascending),
// 10 bits each, the first id most significant; order = ascending signature,
// then ascending block index.  One CTA per (batch*head); rank by counting.
struct OrderParams {
  const int* sel;  // [BH][n_qblk][topk]
  int* order;      // [BH][n_qblk]
  int n_qblk, topk;
};

constexpr int kOrderIds = 6;
constexpr int kOrderMaxQblk = 4096;  // signatures of one (batch, head) in shared memory

__global__ void __launch_bounds__(256) order_kernel(const OrderParams p) {
  extern __shared__ unsigned long long sig[];
  griddep_wait();  // the selection kernel before this one on the stream has completed
  const int s = blockIdx.x;
  const int* rows = p.sel + (size_t)s * p.n_qblk * p.topk;
  for (int j = threadIdx.x; j < p.n_qblk; j += blockDim.x) {
    unsigned long long key = 0ull;
#pragma unroll
    for (int e = 0; e < kOrderIds; ++e) {
      const unsigned id = e < p.topk ? (unsigned)rows[(size_t)j * p.topk + e] & 1023u : 0u;
      key = (key << 10) | id;
    }
    sig[j] = key;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < p.n_qblk; j += blockDim.x) {
    const unsigned long long kj = sig[j];
    int rank = 0;
#pragma unroll 8
    for (int i = 0; i < p.n_qblk; ++i) {
      const unsigned long long ki = sig[i];
      rank += (ki < kj || (ki == kj && i < j)) ? 1 : 0;
    }
    p.order[(size_t)s * p.n_qblk + rank] = j;
  }
}

bool launch_order(const int* sel, int* order, int BH, int n_qblk, int topk, cudaStream_t st) {
  OrderParams op;
  op.sel = sel;
  op.order = order;
  op.n_qblk = n_qblk;
  op.topk = topk;
  // programmatic dependent launch: set-up overlaps the selection kernel
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(BH);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = (size_t)n_qblk * sizeof(unsigned long long);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, order_kernel, op) == cudaSuccess;
}

// The selection kernel, as a programmatic dependent of the window pooling kernel
// when one runs just before it (`after_pool`), else as an ordinary launch.
template <int D>
bool launch_select_t(dim3 g, bool after_pool, cudaStream_t st, const SelParams& sp) {
  static std::mutex mu;
  static unsigned long long attr_done = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && !(attr_done & (1ull << dev))) {
      if (cudaFuncSetAttribute(select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)sel_smem_bytes<D>(kSelStageBytes / (D * 4), true)) != cudaSuccess)
        return false;
      attr_done |= 1ull << dev;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = g;
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = sel_smem_bytes<D>(sp.n_win, sp.stage != 0);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_pool ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, select_kernel<D>, sp) == cudaSuccess;
}

bool launch_select(int d, dim3 g, bool after_pool, cudaStream_t st, const SelParams& sp) {
  return d == 128 ? launch_select_t<128>(g, after_pool, st, sp) : launch_select_t<64>(g, after_pool, st, sp);
}

}  // namespace
}  // namespace vkv

using namespace vkv;

extern "C" vkv_status vkv_block_order(const int32_t* sel_idx, int32_t* out_order, int32_t BH, int32_t n_qblk,
                                      int32_t topk, vkv_stream_t stream) {
  if (!sel_idx || !out_order) return VKV_ERR_NULL;
  if (BH <= 0 || n_qblk <= 0 || topk <= 0) return VKV_ERR_SHAPE;
  if (n_qblk > kOrderMaxQblk || BH > 0x7FFFFFFF / n_qblk) return VKV_ERR_UNSUPPORTED;
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  return launch_order(sel_idx, out_order, BH, n_qblk, topk, reinterpret_cast<cudaStream_t>(stream)) ? VKV_OK
                                                                                                    : VKV_ERR_CUDA;
}

extern "C" size_t vkv_block_select_workspace_size(int32_t B, int32_t H, int32_t Lq, int32_t n_win_blk,
                                                  int32_t block, int32_t d) {
  if (B <= 0 || H <= 0 || Lq <= 0 || n_win_blk <= 0 || block <= 0 || d <= 0) return 0;
  // the window block means; the query blocks are pooled in shared memory
  const size_t bytes = (size_t)B * H * (size_t)n_win_blk * d * sizeof(float);
  return (bytes + 255) & ~(size_t)255;
}

namespace vkv {
namespace {

// Argument checks shared by both selection entry points (workspace excluded).
vkv_status check_select_args(const vkv_select_args* a) {
  if (!a) return VKV_ERR_NULL;
  if (a->d != 64 && a->d != 128) return VKV_ERR_UNSUPPORTED;
  if (a->block != 64) return VKV_ERR_UNSUPPORTED;
  if (a->B <= 0 || a->H <= 0 || a->Lq <= 0 || a->Lkv <= 0) return VKV_ERR_SHAPE;
  if (a->n_win_blk < 1 || a->n_win_blk > 1024 || a->topk < 1 || a->topk > a->n_win_blk) return VKV_ERR_SHAPE;
  if (a->window_blk0 < 0 || (long long)(a->window_blk0 + a->n_win_blk) * a->block > a->Lkv) return VKV_ERR_RANGE;
  if (!a->q.ptr || (!a->k.ptr && !a->kbar) || !a->out_idx) return VKV_ERR_NULL;
  if (!tensor_aligned(a->q) || (!a->kbar && !tensor_aligned(a->k))) return VKV_ERR_ALIGN;
  if (a->kbar && (reinterpret_cast<uintptr_t>(a->kbar) & 15u)) return VKV_ERR_ALIGN;
  if ((long long)a->B * a->H > 65535) return VKV_ERR_UNSUPPORTED;
  if (a->out_order && (a->Lq + a->block - 1) / a->block > kOrderMaxQblk) return VKV_ERR_UNSUPPORTED;
  return VKV_OK;
}

// Window pooling (unless the caller passes cached block means), then scoring
// and top-K (the query blocks are pooled inside the selection kernel), and the
// optional query-block order, on `st`; `kbar_scratch` receives the window
// block means.
vkv_status run_select(const vkv_select_args* a, float* kbar_scratch, cudaStream_t st) {
  const int BH = a->B * a->H;
  const int n_qblk = (a->Lq + 63) / 64;
  const bool pool_win = a->kbar == nullptr;
  if (pool_win) {
    PoolParams pp;
    std::memset(&pp, 0, sizeof(pp));
    pp.k = reinterpret_cast<const __nv_bfloat16*>(a->k.ptr);
    pp.k_sb = a->k.sb; pp.k_st = a->k.st; pp.k_sh = a->k.sh;
    pp.B = a->B;
    pp.H = a->H;
    pp.d = a->d;
    pp.n_qblk = 0;
    pp.n_win = a->n_win_blk;
    pp.win_row0 = a->window_blk0 * a->block;
    pp.kbar = kbar_scratch;
    const int ph = a->d == 128 ? pool_heads<128>() : pool_heads<64>();
    const dim3 pg(a->n_win_blk, a->B * ((a->H + ph - 1) / ph));
    if (a->d == 128)
      pool_kernel<128><<<pg, 256, 0, st>>>(pp);
    else
      pool_kernel<64><<<pg, 256, 0, st>>>(pp);
    if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  }
  SelParams sp;
  sp.q = reinterpret_cast<const __nv_bfloat16*>(a->q.ptr);
  sp.q_sb = a->q.sb; sp.q_st = a->q.st; sp.q_sh = a->q.sh;
  sp.kbar = pool_win ? kbar_scratch : a->kbar;
  sp.H = a->H;
  sp.Lq = a->Lq;
  sp.n_qblk = n_qblk;
  sp.n_win = a->n_win_blk;
  sp.topk = a->topk;
  sp.out_idx = a->out_idx;
  sp.out_scores = a->out_scores;
  sp.err = a->err_word;
  // the head's window means are staged in shared memory when they fit (16-byte
  // aligned source: every head's block holds n_win * d floats)
  const size_t wbytes = (size_t)a->n_win_blk * (a->d + 4) * sizeof(float);
  sp.stage = (wbytes <= (size_t)kSelStageBytes && (reinterpret_cast<uintptr_t>(sp.kbar) & 15u) == 0) ? 1 : 0;
  const dim3 sg((n_qblk + kSelQ - 1) / kSelQ, BH);
  if (!launch_select(a->d, sg, pool_win, st, sp)) return VKV_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  if (a->out_order && !launch_order(a->out_idx, a->out_order, BH, n_qblk, a->topk, st)) return VKV_ERR_CUDA;
  return VKV_OK;
}

}  // namespace
}  // namespace vkv

extern "C" vkv_status vkv_block_select(const vkv_select_args* a, vkv_stream_t stream) {
  const vkv_status chk = check_select_args(a);
  if (chk != VKV_OK) return chk;
  // the workspace holds the window block means, so it is needed only when they are pooled here
  if (!a->kbar) {
    const size_t need = vkv_block_select_workspace_size(a->B, a->H, a->Lq, a->n_win_blk, a->block, a->d);
    if (!a->workspace || a->workspace_bytes < need) return VKV_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(a->workspace) & 255u) return VKV_ERR_ALIGN;
  }
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  return run_select(a, reinterpret_cast<float*>(a->workspace), reinterpret_cast<cudaStream_t>(stream));
}

extern "C" vkv_status vkv_block_pool(vkv_tensor x, int32_t B, int32_t L, int32_t H, int32_t d, int32_t blk0,
                                     int32_t n_blk, float* out, vkv_stream_t stream) {
  if (!x.ptr || !out) return VKV_ERR_NULL;
  if (d != 64 && d != 128) return VKV_ERR_UNSUPPORTED;
  if (B <= 0 || H <= 0 || L <= 0 || n_blk <= 0 || blk0 < 0) return VKV_ERR_SHAPE;
  if ((long long)(blk0 + n_blk) * 64 > L) return VKV_ERR_RANGE;
  if (!tensor_aligned(x) || (reinterpret_cast<uintptr_t>(out) & 15u)) return VKV_ERR_ALIGN;
  if ((long long)B * H > 65535) return VKV_ERR_UNSUPPORTED;
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  // the window-block path of the selection's pooling kernel, with no query blocks
  PoolParams pp;
  std::memset(&pp, 0, sizeof(pp));
  pp.k = reinterpret_cast<const __nv_bfloat16*>(x.ptr);
  pp.k_sb = x.sb; pp.k_st = x.st; pp.k_sh = x.sh;
  pp.B = B;
  pp.H = H;
  pp.d = d;
  pp.Lq = 0;
  pp.n_qblk = 0;
  pp.n_win = n_blk;
  pp.win_row0 = blk0 * 64;
  pp.kbar = out;
  const int ph = d == 128 ? pool_heads<128>() : pool_heads<64>();
  const dim3 pg(n_blk, B * ((H + ph - 1) / ph));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128)
    pool_kernel<128><<<pg, 256, 0, st>>>(pp);
  else
    pool_kernel<64><<<pg, 256, 0, st>>>(pp);
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
// For them the pooled window block vectors live in one file-scope device
// array of fixed size, kNoallocScratchBytes, which every GPU that loads the
// library holds until the process exits (calls that pass cached window means
// in `kbar` do not use it).
//
// In host code `g_select_scratch` is only a host-side stand-in for the array;
// its device address is looked up once per device (cudaGetSymbolAddress, with
// that device current) on the first call made on it, and cached.  The cached
// address belongs to the device's context at that time: after a
// cudaDeviceReset the entry point must not be called again in the process.
// Every call on a device shares the array and leaves the last call's contents
// behind; nothing needs clearing, because every element the select kernel
// reads is written by the pool kernel of the same call.  Calls that overlap on
// the GPU (for example on two streams at once) race on the array.
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
  const vkv_status chk = check_select_args(a);
  if (chk != VKV_OK) return chk;
  // the scratch holds the window block means, which cached representatives (kbar) replace
  const size_t need =
      a->kbar ? 0 : vkv_block_select_workspace_size(a->B, a->H, a->Lq, a->n_win_blk, a->block, a->d);
  if (need > kNoallocScratchBytes) return VKV_ERR_WORKSPACE;  // larger than the fixed scratch array
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  void* scratch = noalloc_scratch(dev);
  if (!scratch) return VKV_ERR_CUDA;
  return run_select(a, reinterpret_cast<float*>(scratch), reinterpret_cast<cudaStream_t>(stream));
}
