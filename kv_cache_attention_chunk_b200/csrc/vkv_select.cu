// vkv_block_select: blockified coarse scoring and top-K window-block selection
// (Sparse Forcing summary, section 2 component 2 "Blockified Compression": one
// representative token per block for coarse scoring; component 3 "PBSA":
// top-K blocks of the local window, per query block).
//
// Two kernels on the caller's stream:
//   pool_kernel     mean of every 64-row block of Q and of the window part of K,
//                   in fp32, written to the caller's workspace.  One CTA of 256
//                   threads per (block, batch, group of 512/d heads): the group's
//                   contiguous slice of each row is read with 16-byte loads,
//                   16 rows per thread in flight; row groups are combined in
//                   shared memory.  HBM-bound.
//   select_kernel   one CTA per (batch*head, 8 query blocks): the pooled keys
//                   are copied to shared memory 160 blocks at a time (cp.async),
//                   each thread scores one window block against the CTA's eight
//                   pooled queries, then one warp per query block runs an exact
//                   top-K: radix selection of the K-th largest score on
//                   order-preserving keys, ties at the threshold to the lower
//                   block index; kept blocks are written in ascending order.
//                   Launched as a programmatic dependent of the pooling kernel,
//                   so its launch overlaps the pooling kernel's last CTAs.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "vkv_internal.h"
#include "vkv_pool.cuh"
#include "vkv_ptx.cuh"

namespace vkv {

// Development timeline (compiled only with -DVKV_TRACE): clock stamps of the
// phases of select CTA (0, 0), read back with vkv_debug_sel_trace().
#ifdef VKV_TRACE
__device__ unsigned long long g_vkv_sel_trace[64];
#define VKV_SEL_STAMP(i)                                                              \
  do {                                                                                \
    if (blockIdx.x == 0 && blockIdx.y == 0 && (threadIdx.x & 31) == 0)               \
      g_vkv_sel_trace[(threadIdx.x >> 5) * 8 + (i)] = clock64();                     \
  } while (0)
#else
#define VKV_SEL_STAMP(i) \
  do {                   \
  } while (0)
#endif

namespace {

struct SelParams {
  const float* qbar;
  const float* kbar;
  int BH, n_qblk, n_win, topk;
  int* out_idx;
  float* out_scores;
};

constexpr int kSelWarps = 8;     // query blocks per CTA (one warp each for the top-K)
constexpr int kSelChunk = 160;   // window blocks staged in shared memory at a time

template <int D>
__host__ __device__ constexpr int sel_row_stride() { return D + 4; }  // floats; keeps rows 16-byte aligned

template <int D>
constexpr size_t sel_smem_bytes(int n_win) {
  return ((size_t)kSelWarps * D + (size_t)kSelChunk * sel_row_stride<D>() + (size_t)kSelWarps * n_win) *
         sizeof(float);
}
constexpr int kSelMaxSmem = (int)sel_smem_bytes<128>(1024);

// grid: x = ceil(n_qblk / kSelWarps), y = b*H + h; 32 * kSelWarps threads.
// Shared memory: the CTA's pooled queries [kSelWarps][D], a chunk of pooled
// keys [kSelChunk][D + 4] and the scores [kSelWarps][n_win].  Pooled vectors
// are copied with cp.async (every copy of a chunk in flight at once).  Thread i
// scores window block w0 + i against all of the CTA's pooled queries: its key
// row is read from shared memory once (float4 reads; with the 4-float pad the
// eight rows of a quarter warp fall in distinct banks), the query rows are
// broadcast.  Then warp q selects the top-K of query block j0 + q.
template <int D, int kMaxPerLane>
__global__ void __launch_bounds__(32 * kSelWarps) select_kernel(const SelParams p) {
  extern __shared__ __align__(16) float sm[];
  constexpr int RS = sel_row_stride<D>();
  constexpr int D4 = D / 4;
  float* qs = sm;                              // kSelWarps * D
  float* ks = qs + kSelWarps * D;              // kSelChunk * RS
  float* scs = ks + kSelChunk * RS;            // kSelWarps * n_win
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int s = blockIdx.y;
  const int j0 = blockIdx.x * kSelWarps;
  const int nq = min(kSelWarps, p.n_qblk - j0);
  const int j = j0 + warp;
  const bool active = warp < nq;
  VKV_SEL_STAMP(0);
  griddep_launch_dependents();  // the (small) order kernel may be scheduled alongside
  griddep_wait();  // the pooling kernel before this one on the stream has completed
  VKV_SEL_STAMP(1);
  const float* qsrc = p.qbar + ((size_t)s * p.n_qblk + j0) * D;
  for (int x = threadIdx.x; x < kSelWarps * D4; x += blockDim.x) {
    if (x < nq * D4)
      cp_async16(qs + 4 * x, qsrc + 4 * x);
    else
      reinterpret_cast<float4*>(qs)[x] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float* kb = p.kbar + (size_t)s * p.n_win * D;
  for (int w0 = 0; w0 < p.n_win; w0 += kSelChunk) {
    const int nw = min(kSelChunk, p.n_win - w0);
    __syncthreads();  // the previous chunk is fully consumed
    for (int x = threadIdx.x; x < nw * D4; x += blockDim.x) {
      const int r = x / D4, c4 = x - (x / D4) * D4;
      cp_async16(ks + r * RS + 4 * c4, kb + (size_t)(w0 + r) * D + 4 * c4);
    }
    cp_async_wait_all();
    __syncthreads();
    VKV_SEL_STAMP(2);
    for (int r = threadIdx.x; r < nw; r += blockDim.x) {
      const float4* kr = reinterpret_cast<const float4*>(ks + r * RS);
      float acc[kSelWarps][4];
#pragma unroll
      for (int q = 0; q < kSelWarps; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.f;
#pragma unroll 4
      for (int c = 0; c < D4; ++c) {
        const float4 kv = kr[c];
#pragma unroll
        for (int q = 0; q < kSelWarps; ++q) {
          const float4 qv = reinterpret_cast<const float4*>(qs + q * D)[c];
          acc[q][0] = fmaf(qv.x, kv.x, acc[q][0]);
          acc[q][1] = fmaf(qv.y, kv.y, acc[q][1]);
          acc[q][2] = fmaf(qv.z, kv.z, acc[q][2]);
          acc[q][3] = fmaf(qv.w, kv.w, acc[q][3]);
        }
      }
#pragma unroll
      for (int q = 0; q < kSelWarps; ++q) {
        const float v = (acc[q][0] + acc[q][1]) + (acc[q][2] + acc[q][3]);
        // NaN ranks last; -0 becomes +0 so that equal scores tie on the block index
        scs[q * p.n_win + w0 + r] = (v != v) ? -INFINITY : (v == 0.f ? 0.f : v);
      }
    }
  }
  __syncthreads();
  VKV_SEL_STAMP(3);
  const float* sc = scs + warp * p.n_win;
  if (!active) return;
  if (p.out_scores) {
    float* so = p.out_scores + ((size_t)s * p.n_qblk + j) * p.n_win;
    for (int w = lane; w < p.n_win; w += 32) so[w] = sc[w];
  }
  // exact top-K by radix selection of the topk-th largest score on
  // order-preserving integer keys (32 rounds); every block above that
  // score is kept, and of the blocks equal to it the lowest indices are kept.
  // Each lane owns blocks w = lane + 32m.
  const int per = (p.n_win + 31) >> 5;  // <= kMaxPerLane
  uint32_t key[kMaxPerLane];
#pragma unroll
  for (int m = 0; m < kMaxPerLane; ++m) {
    const int w = lane + 32 * m;
    if (m < per && w < p.n_win) {
      const uint32_t u = __float_as_uint(sc[w]);
      key[m] = u ^ ((u >> 31) ? 0xFFFFFFFFu : 0x80000000u);  // larger score -> larger key
    } else {
      key[m] = 0u;  // absent: below every real score (whose keys are >= 0x007FFFFF)
    }
  }
  uint32_t prefix = 0u, mask = 0u;
  int need = p.topk;  // rank, among the not-yet-excluded keys, of the threshold
  // one bit per round, most significant first (one warp sum per round: warp
  // collectives are the cost here, so the fewest of them wins)
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t want = prefix | (1u << bit), mk = mask | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int m = 0; m < kMaxPerLane; ++m)
      if (m < per) cnt += ((key[m] & mk) == want) ? 1 : 0;
    cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
    if (cnt >= need) {
      prefix = want;
    } else {
      need -= cnt;
    }
    mask = mk;
  }
  VKV_SEL_STAMP(4);
  // prefix = key of the topk-th largest score; `need` of its equals are kept
  int* oi = p.out_idx + ((size_t)s * p.n_qblk + j) * p.topk;
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int m = 0; m < kMaxPerLane; ++m) {
    if (m < per) {
      const int w = lane + 32 * m;
      const bool valid = w < p.n_win;
      const bool eq = valid && key[m] == prefix;
      const uint32_t beq = __ballot_sync(0xFFFFFFFFu, eq);
      const int eq_rank = eq_seen + __popc(beq & ((1u << lane) - 1u));
      const bool keep = valid && (key[m] > prefix || (eq && eq_rank < need));
      eq_seen += __popc(beq);
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
      if (keep) oi[written + __popc(bal & ((1u << lane) - 1u))] = w;
      written += __popc(bal);
    }
  }
  VKV_SEL_STAMP(5);
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

// Instantiation by head dimension and by window size (candidates per lane).
template <int D, int PER>
bool launch_select_t(dim3 g, size_t smem, cudaStream_t st, const SelParams& sp) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(select_kernel<D, PER>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelMaxSmem) !=
        cudaSuccess)
      return false;
    attr_set[dev] = true;
  }
  // programmatic dependent launch: set-up overlaps the tail of the pooling kernel
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = g;
  cfg.blockDim = dim3(32 * kSelWarps);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_kernel<D, PER>, sp) == cudaSuccess;
}

template <int D>
bool launch_select_d(int n_win, dim3 g, size_t smem, cudaStream_t st, const SelParams& sp) {
  if (n_win <= 160) return launch_select_t<D, 5>(g, smem, st, sp);
  if (n_win <= 256) return launch_select_t<D, 8>(g, smem, st, sp);
  if (n_win <= 512) return launch_select_t<D, 16>(g, smem, st, sp);
  return launch_select_t<D, 32>(g, smem, st, sp);
}

bool launch_select(int d, int n_win, dim3 g, size_t smem, cudaStream_t st, const SelParams& sp) {
  return d == 128 ? launch_select_d<128>(n_win, g, smem, st, sp) : launch_select_d<64>(n_win, g, smem, st, sp);
}

}  // namespace
}  // namespace vkv

using namespace vkv;

#ifdef VKV_TRACE
// Development only (not in the public header): copy select CTA (0, 0)'s stamps.
extern "C" int vkv_debug_sel_trace(void* dst, size_t bytes) {
  cudaDeviceSynchronize();
  return (int)cudaMemcpyFromSymbol(dst, vkv::g_vkv_sel_trace,
                                   bytes < sizeof(vkv::g_vkv_sel_trace) ? bytes : sizeof(vkv::g_vkv_sel_trace));
}
#endif

extern "C" size_t vkv_block_select_workspace_size(int32_t B, int32_t H, int32_t Lq, int32_t n_win_blk,
                                                  int32_t block, int32_t d) {
  if (B <= 0 || H <= 0 || Lq <= 0 || n_win_blk <= 0 || block <= 0 || d <= 0) return 0;
  const size_t n_qblk = (size_t)(Lq + block - 1) / block;
  const size_t bytes = (size_t)B * H * (n_qblk + (size_t)n_win_blk) * d * sizeof(float);
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

// Pooling (query blocks, and the window blocks unless cached), scoring and
// top-K, and the optional query-block order, on `st`; `scratch` holds the
// pooled vectors.
vkv_status run_select(const vkv_select_args* a, float* scratch, cudaStream_t st) {
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
  pp.qbar = scratch;
  pp.kbar = pp.qbar + (size_t)BH * n_qblk * a->d;
  const int ph = a->d == 128 ? pool_heads<128>() : pool_heads<64>();
  // with cached window representatives only the query blocks are pooled
  const dim3 pg(n_qblk + (a->kbar ? 0 : a->n_win_blk), a->B * ((a->H + ph - 1) / ph));
  if (a->d == 128)
    pool_kernel<128><<<pg, 256, 0, st>>>(pp);
  else
    pool_kernel<64><<<pg, 256, 0, st>>>(pp);
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  SelParams sp;
  sp.qbar = pp.qbar;
  sp.kbar = a->kbar ? a->kbar : pp.kbar;
  sp.BH = BH;
  sp.n_qblk = n_qblk;
  sp.n_win = a->n_win_blk;
  sp.topk = a->topk;
  sp.out_idx = a->out_idx;
  sp.out_scores = a->out_scores;
  const dim3 sg((n_qblk + kSelWarps - 1) / kSelWarps, BH);
  const size_t smem = a->d == 128 ? sel_smem_bytes<128>(a->n_win_blk) : sel_smem_bytes<64>(a->n_win_blk);
  if (!launch_select(a->d, a->n_win_blk, sg, smem, st, sp)) return VKV_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  if (a->out_order && !launch_order(a->out_idx, a->out_order, BH, n_qblk, a->topk, st)) return VKV_ERR_CUDA;
  return VKV_OK;
}

}  // namespace
}  // namespace vkv

extern "C" vkv_status vkv_block_select(const vkv_select_args* a, vkv_stream_t stream) {
  const vkv_status chk = check_select_args(a);
  if (chk != VKV_OK) return chk;
  const size_t need = vkv_block_select_workspace_size(a->B, a->H, a->Lq, a->n_win_blk, a->block, a->d);
  if (!a->workspace || a->workspace_bytes < need) return VKV_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(a->workspace) & 255u) return VKV_ERR_ALIGN;
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
  const vkv_status chk = check_select_args(a);
  if (chk != VKV_OK) return chk;
  const size_t need = vkv_block_select_workspace_size(a->B, a->H, a->Lq, a->n_win_blk, a->block, a->d);
  if (need > kNoallocScratchBytes) return VKV_ERR_WORKSPACE;  // larger than the fixed scratch array
  int dev = 0;
  if (device_sm_count(&dev) <= 0) return VKV_ERR_CUDA;
  void* scratch = noalloc_scratch(dev);
  if (!scratch) return VKV_ERR_CUDA;
  return run_select(a, reinterpret_cast<float*>(scratch), reinterpret_cast<cudaStream_t>(stream));
}
