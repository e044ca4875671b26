// Chunk attention over a segmented KV cache: the sm_100a kernel.
//
// One persistent CTA per SM works through a host-built list of units.  A
// unit is one (batch, head) and one or two 128-row query tiles; it walks a
// stream of 128-key tiles (two 64-row halves each) and keeps an online
// softmax per query row.  The key stream depends on the mode:
//   SEGMENTS      consecutive 128-row tiles of each segment of each branch
//                 (ISPA summary, section 2 step 1: local and history branches,
//                 each closed with its own output and LSE, then merged);
//   BLOCK_SPARSE  the unit's persistent blocks, then the union of the window
//                 blocks selected for its four 64-query blocks (consecutive in
//                 the caller's query-block order, which may group blocks with
//                 similar selections), two blocks per tile, with a per-query-
//                 block visibility mask (Sparse Forcing summary, section 2
//                 component 3 "PBSA");
//   RAGGED        consecutive tiles of rows [cu[s], cu[s+1]) of the flattened
//                 cache (Pyramid Forcing summary, methodology section 3).
//
// Warp roles (384 threads):
//   warp 0       TMA producer: Q tiles, K/V tiles into a ring of smem slots.
//   warp 1       MMA issuer: S_t = Q_t K^T and O_t += P_t V with tcgen05.mma,
//                accumulators in tensor memory (TMEM); owns the TMEM allocation.
//   warps 2-3    BLOCK_SPARSE: warp 2 builds each unit's block list from the
//                caller's selection, one unit ahead of the other roles; or, with
//                the selection in the kernel (FS), warps 2-3 select the window
//                blocks themselves.  Idle in the other modes.
// With key-axis pieces (PC), a piece leaves fp32 partials in a workspace and
// piece_combine_kernel, launched behind this grid, merges them.
//   warps 4-7    softmax + epilogue for query tile 0 (one thread per row).
//   warps 8-11   softmax + epilogue for query tile 1.
// In the selecting (FS) kernel a one-tile unit gives its even key steps to
// warps 4-7 (S_0, O_0) and its odd ones to warps 8-11 (S_1, O_1); the two
// partial states are merged by their LSEs at the end of the unit.
//
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 [256+D,256+2D).
// The softmax threads read S_t, then write P_t (bf16, two per 32-bit column)
// over the first 64 columns of S_t; the PV MMA reads P_t from TMEM (A operand)
// and V from shared memory.  Per tile the MMA thread issues O_t += P_t(j) V_j
// before S_t(j+1) = Q_t K_{j+1}^T, so P_t(j) is consumed before S_t is
// overwritten (tcgen05.mma ops of one thread execute in issue order).
// Keeping P out of shared memory leaves room for a 5-slot K/V ring (d = 128).
// The online softmax works in log2 units (s * scale * log2 e) and rescales the
// O accumulator only when a row maximum grows by more than 2^8; the final
// O / l and LSE do not depend on the reference maximum.
#pragma once

#include "vkv_internal.h"
#include "vkv_ptx.cuh"
#include "vkv_topk.cuh"

namespace vkv {

template <int D>
struct AttnCfg {
  static constexpr int NAC = D / 64;               // 128-byte atom columns along d
  static constexpr int ATOM = 128 * 128;            // bytes of one 128-row atom column
  static constexpr int QT_BYTES = 128 * D * 2;      // one 128-row Q tile
  static constexpr int KV_BYTES = 128 * D * 2;      // one K or V tile (128 keys)
  static constexpr int NSLOT = (D == 128) ? 5 : 8;  // K/V ring slots
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + 2 * QT_BYTES;
  static constexpr int OFF_CTL = OFF_KV + NSLOT * KV_BYTES;
  static constexpr int SMEM_BYTES = OFF_CTL + kCtlBytes + 1024;  // + base alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_O = 256;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

constexpr int kMaxSlots = 8;

// Control block (barriers, block list) at the end of shared memory.
struct Ctl {
  uint64_t full[kMaxSlots];
  uint64_t empty[kMaxSlots];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t list_ready[2], list_free[2], drain;  // one pair per block-list buffer
  uint64_t list_pers[2];  // FS: the buffer's persistent prefix is written
  uint32_t tmem_base;
  int abort_flag;
  int list_count[2];
  int pers_count[2];  // FS: entries of the persistent prefix
  int sel_go;         // FS: the selection warps may write the next list buffer
  uint32_t bitmap[4][32];
  uint32_t list[kMaxListEntries];  // block-list buffer 0 (buffer 1: the ring's last K/V slot)
  uint64_t kx_sync;  // FS one-tile unit split over both warpgroups: states written, then read
};
static_assert(sizeof(Ctl) <= kCtlBytes, "control block");

struct TileDesc {
  int rowA, rowB;         // first cache row of each 64-row half
  int limA, limB;         // valid columns of each half (0..64)
  uint32_t maskA, maskB;  // per-64-query-block visibility bits of each half
  int branch;
  bool first;             // first tile of its branch
};

// Walks the key-tile stream of one unit; every role runs its own copy.
struct TileIter {
  const AttnParams* p;
  const uint32_t* list;  // BLOCK_SPARSE: the unit's block list and its length
  int count;
  int k, off;        // SEGMENTS: flat segment index, row offset inside it
  int rstart, rlen;  // RAGGED: this sequence's rows
  int j;

  __device__ __forceinline__ void init(const AttnParams* pp, const uint32_t* lst, int cnt, int rs, int rl) {
    p = pp;
    list = lst;
    count = cnt;
    k = 0;
    off = 0;
    rstart = rs;
    rlen = rl;
    j = 0;
  }

  // Start the walk at key-tile step j0 (a piece of a split unit); SEGMENTS and
  // RAGGED only, with j0 below the unit's step count.
  __device__ __forceinline__ void seek(int j0) {
    if (p->mode == VKV_MODE_SEGMENTS) {
      int kk = 0;
      while (kk + 1 < p->n_flat && p->flat_step0[kk + 1] <= j0) ++kk;
      k = kk;
      off = (j0 - p->flat_step0[kk]) * 128;
    } else {
      off = j0 * 128;
    }
    j = j0;
  }

  __device__ __forceinline__ TileDesc next() {
    TileDesc t;
    if (p->mode == VKV_MODE_BLOCK_SPARSE) {
      const int n = count;
      const uint32_t e0 = list[2 * j];
      const uint32_t e1 = (2 * j + 1 < n) ? list[2 * j + 1] : (e0 & 0xFFFFFFu);
      t.rowA = (int)(e0 & 0xFFFFFFu) * 64;
      t.rowB = (int)(e1 & 0xFFFFFFu) * 64;
      t.limA = 64;
      t.limB = 64;
      t.maskA = e0 >> 24;
      t.maskB = e1 >> 24;
      t.branch = 0;
      t.first = (j == 0);
    } else {
      int start, len, br;
      bool bfirst;
      if (p->mode == VKV_MODE_RAGGED) {
        start = rstart;
        len = rlen;
        br = 0;
        bfirst = true;
      } else {
        start = p->flat_start[k];
        len = p->flat_len[k];
        br = p->flat_branch[k];
        bfirst = p->flat_first[k] != 0;
      }
      const int valid = min(128, len - off);
      t.rowA = start + off;
      t.rowB = start + off + 64;
      t.limA = min(64, valid);
      t.limB = max(0, valid - 64);
      t.maskA = 0xFu;
      t.maskB = 0xFu;
      t.branch = br;
      t.first = bfirst && off == 0;
      off += 128;
      if (off >= len) {
        ++k;
        off = 0;
      }
    }
    ++j;
    return t;
  }
};

struct UnitInfo {
  int s;       // sequence = b*H + h
  int b, h;
  int tile0;   // first 128-row query tile
  int ntiles;  // 1 or 2
  bool piece;  // covers only the key steps of its piece entry
};

struct PieceInfo {
  int j0, j1;  // key-tile steps [j0, j1) of the unit's stream
  int slot0;   // the unit's first workspace slot (its counters live there)
  int idx, n;  // this piece's index and the unit's piece count
};

__device__ __forceinline__ PieceInfo piece_info(const AttnParams& p, int k) {
  const uint2 e = p.pieces[k];
  PieceInfo r;
  r.j0 = (int)(e.x & 0xFFFFu);
  r.j1 = (int)(e.x >> 16);
  r.slot0 = (int)(e.y & 0xFFFFu);
  r.idx = (int)((e.y >> 16) & 0xFFu);
  r.n = (int)(e.y >> 24);
  return r;
}

// Steps of this unit entry: all `full` steps of the unit's stream, or the part
// [j0, j1) of a piece (pi.j0 is set to the entry's first step).  RAGGED
// lengths are read on the device and may differ from the host copy the pieces
// were cut from: the range is clamped to `full`, and the unit's last piece
// runs to `full`, so the pieces always cover the device's key range.  A
// BLOCK_SPARSE unit's step count is known only on the device: its pieces were
// cut from the host's estimate sp_est[ntiles - 1] and are scaled to `full`.
// Advances the CTA's piece cursor; every role walks the same unit list.
__device__ __forceinline__ int entry_steps(const AttnParams& p, const UnitInfo& u, int full, int& piece_k,
                                           PieceInfo& pi) {
  if (!u.piece) {
    pi.j0 = 0;
    pi.n = 0;
    return full;
  }
  pi = piece_info(p, piece_k++);
  const bool last = pi.idx == pi.n - 1;
  if (p.mode == VKV_MODE_BLOCK_SPARSE) {
    const int est = max(1, p.sp_est[u.ntiles - 1]);
    pi.j0 = (int)(((long long)pi.j0 * full) / est);
    pi.j1 = last ? full : (int)(((long long)pi.j1 * full) / est);
    return max(0, min(pi.j1, full) - pi.j0);
  }
  const int j1 = last ? full : min(pi.j1, full);
  return max(0, j1 - pi.j0);
}

__device__ __forceinline__ UnitInfo decode_unit(const AttnParams& p, uint32_t code) {
  UnitInfo u;
  u.tile0 = (int)(code & 0xFFFu);
  u.piece = ((code >> 12) & 1u) != 0;
  u.ntiles = ((code >> 13) & 1u) ? 2 : 1;
  u.s = (int)(code >> 14);
  u.b = u.s / p.H;
  u.h = u.s - u.b * p.H;
  return u;
}

// A unit entry as the kernel instantiation sees it: without piece support (PC
// false) no entry is a piece, and every piece path folds away at compile time.
template <bool PC>
__device__ __forceinline__ UnitInfo decode_entry(const AttnParams& p, uint32_t code) {
  UnitInfo u = decode_unit(p, code);
  if (!PC) u.piece = false;
  return u;
}

__device__ __forceinline__ void set_err(const AttnParams& p, int code) {
  if (p.err) atomicCAS(p.err, 0, code);
}

// BLOCK_SPARSE: query block at position `pos` of sequence s's unit order
// (qblk_order, or the natural order); -1 past the last block.  An entry out of
// range records VKV_DEVERR_BAD_INDEX and falls back to the natural order.
__device__ __forceinline__ int unit_qblk(const AttnParams& p, int s, int pos, bool report) {
  if (pos >= p.n_qblk) return -1;
  if (!p.qblk_order) return pos;
  const int q = __ldg(p.qblk_order + (size_t)s * p.n_qblk + pos);
  if (q < 0 || q >= p.n_qblk) {
    if (report) set_err(p, VKV_DEVERR_BAD_INDEX);
    return pos;
  }
  return q;
}

// Rows [start, start+len) of a ragged sequence, checked on the device.
__device__ __forceinline__ void ragged_range(const AttnParams& p, int s, int& start, int& len,
                                             bool report) {
  const int a = __ldg(p.cu_seqlens + s);
  const int b = __ldg(p.cu_seqlens + s + 1);
  if (a < 0 || b < a || b > p.Lkv) {
    start = 0;
    len = 0;
    if (report) set_err(p, VKV_DEVERR_BAD_OFFSETS);
  } else {
    start = a;
    len = b - a;
  }
}

__device__ __forceinline__ int unit_steps(const AttnParams& p, int list_count, int rlen) {
  if (p.mode == VKV_MODE_SEGMENTS) return p.total_steps;
  if (p.mode == VKV_MODE_RAGGED) return (rlen + 127) >> 7;
  return (list_count + 1) >> 1;
}

// The persistent blocks of sequence s at the head of a unit's block list (visible
// to all nqb query blocks of the unit); an index outside the cache or inside the
// window records VKV_DEVERR_BAD_INDEX and is skipped.  Returns the entry count.
// Executed by all 32 lanes of one warp.
__device__ __forceinline__ int build_persist_prefix(const AttnParams& p, int s, int nqb, uint32_t* list) {
  const uint32_t lane = lane_id();
  const uint32_t all_mask = (nqb > 0) ? ((1u << nqb) - 1u) : 0u;
  int base = 0;
  const int* prow = p.persist_idx + (size_t)s * p.n_persist;
  for (int e0 = 0; e0 < p.n_persist; e0 += 32) {
    const int e = e0 + (int)lane;
    int blk = -1;
    bool ok = false;
    if (e < p.n_persist) {
      blk = __ldg(prow + e);
      ok = blk >= 0 && blk < p.n_blocks_total &&
           (blk < p.window_blk0 || blk >= p.window_blk0 + p.n_win_blk);
      if (!ok) set_err(p, VKV_DEVERR_BAD_INDEX);
    }
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, ok);
    if (ok) list[base + __popc(bal & ((1u << lane) - 1u))] = (uint32_t)blk | (all_mask << 24);
    base += __popc(bal);
  }
  return base;
}

// The union of the window blocks that the unit's nqb query blocks selected
// (ctl->bitmap[i]: bit w of query block i), ascending, each tagged with the
// query blocks that selected it, appended at list[base]; the list's length goes
// to *list_count.  Executed by all 32 lanes of one warp.
__device__ __forceinline__ void build_window_union(const AttnParams& p, Ctl* ctl, int nqb, uint32_t* list,
                                                   int base, int* list_count) {
  const uint32_t lane = lane_id();
  const int nwords = (p.n_win_blk + 31) >> 5;
  // lane L owns window blocks [32L, 32L + 32)
  uint32_t m[4], uni = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = ((int)lane < nwords && i < nqb) ? ctl->bitmap[i][lane] : 0u;
    uni |= m[i];
  }
  const int cnt = __popc(uni);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if ((int)lane >= o) incl += v;
  }
  const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
  int pos = base + incl - cnt;
  uint32_t rest = uni;
  while (rest) {
    const int bit = __ffs(rest) - 1;
    rest &= rest - 1u;
    uint32_t qm = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) qm |= ((m[i] >> bit) & 1u) << i;
    list[pos++] = (uint32_t)(p.window_blk0 + (int)lane * 32 + bit) | (qm << 24);
  }
  if (lane == 0) *list_count = base + total;
  __threadfence_block();
  __syncwarp();
}

// Build the unit's block list (BLOCK_SPARSE) from the caller's selection:
// persistent blocks (visible to every query block of the unit) followed by the
// union of the window blocks selected by the unit's query blocks, ascending,
// each tagged with the query blocks that selected it.  Executed by all 32
// lanes of one warp.
__device__ __forceinline__ void build_block_list(const AttnParams& p, Ctl* ctl, const UnitInfo& u,
                                                 uint32_t* list, int* list_count) {
  const uint32_t lane = lane_id();
  const int qb0 = u.tile0 * 2;
  const int nqb = min(2 * u.ntiles, p.n_qblk - qb0);
#pragma unroll
  for (int i = 0; i < 4; ++i) ctl->bitmap[i][lane] = 0u;
  __syncwarp();
  for (int i = 0; i < nqb; ++i) {
    const int qbi = unit_qblk(p, u.s, qb0 + i, lane == 0);
    const int* row = p.sel_idx + ((size_t)u.s * p.n_qblk + qbi) * p.topk;
    for (int e = lane; e < p.topk; e += 32) {
      const int w = __ldg(row + e);
      if (w >= 0 && w < p.n_win_blk) {
        atomicOr(&ctl->bitmap[i][w >> 5], 1u << (w & 31));
      } else {
        set_err(p, VKV_DEVERR_BAD_INDEX);
      }
    }
  }
  __syncwarp();
  const int base = build_persist_prefix(p, u.s, nqb, list);
  build_window_union(p, ctl, nqb, list, base, list_count);
}

// ---------------------------------------------------------------------------
// Selection inside the block-sparse kernel (FS instantiation).  Warps 2-3 choose
// the window blocks of each unit's query blocks from the cached window block
// means (Sparse Forcing summary, section 2 component 2 "Blockified
// Compression": one representative per block for coarse scoring) and publish
// the unit's block list in two steps: the persistent prefix at once
// (list_pers), which the other roles start streaming, then the union of the
// selections (list_ready).  The arithmetic follows the standalone selection
// kernel operation for operation -- the same row grouping and addition order of
// the query pooling, the same multiply-add chains of the scores, the same
// warp_topk -- so the choice equals vkv_block_select's with cached means.
// ---------------------------------------------------------------------------
constexpr int kFsMaxWin = 512;  // window blocks the selection keys have room for

// Selection scratch in the block-sparse instantiation's last K/V slot, after the
// second block list: pooled queries [4][D] fp32, one 256-bin histogram per
// selection warp, ranking keys [4][kFsMaxWin].
template <int D>
struct FsScratch {
  static constexpr int OFF_QS = 1280;
  static constexpr int OFF_HIST = OFF_QS + 4 * D * 4;
  static constexpr int OFF_KEYS = OFF_HIST + 2 * 256 * 4;
  static constexpr int BYTES = OFF_KEYS + 4 * kFsMaxWin * 4;
  static_assert(kMaxListEntries * 4 <= OFF_QS, "second block list");
  static_assert(BYTES <= AttnCfg<D>::KV_BYTES, "selection scratch");
};

// A one-tile unit of the selecting (FS) kernel, whose key tiles alternate between
// the two softmax warpgroups, ends with both warpgroups' row states (m, l) side by side,
// float [warpgroup 2][m, l][row 128], at the end of the ring's last K/V slot:
// past the second block list and the selection scratch, and used by one unit
// at a time (a warpgroup leaves the unit only once both have read them).
template <int D>
struct KxScratch {
  static constexpr int OFF = AttnCfg<D>::KV_BYTES - 2048;
  static_assert(FsScratch<D>::BYTES <= OFF, "exchange area after the selection scratch");
};

// Named barrier of the two selection warps.
__device__ __forceinline__ void fs_bar() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

// Mean of each of the unit's nq query blocks (positions qb0 .. qb0 + nq - 1 of
// the unit order) into qs[q][D]: thread
// (q, c) of the 64 sums the 16-byte column chunk c of the block's rows in row
// groups g = 0 .. G-1 (rows g, g + G, ...), group by group, then divides by the
// block's row count -- the standalone kernel's order of additions.
template <int D>
__device__ __forceinline__ void fs_pool(const AttnParams& p, const UnitInfo& u, int qb0, int nq, float* qs,
                                        int st) {
  constexpr int CPR = D / 8, G = 256 / CPR, RPT = 64 / G;
  const __nv_bfloat16* base = p.qp + u.b * p.q_sb + u.h * p.q_sh;
  for (int x = st; x < 4 * CPR; x += 64) {
    const int q = x / CPR, c = x % CPR;
    if (q >= nq) continue;
    const int qb = unit_qblk(p, u.s, qb0 + q, c == 0);
    float sum[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sum[e] = 0.f;
#pragma unroll 1
    for (int g0 = 0; g0 < G; g0 += 2) {
      uint4 v[2][RPT];
#pragma unroll
      for (int gi = 0; gi < 2; ++gi)
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
          const int row = qb * 64 + g0 + gi + G * i;
          v[gi][i] = row < p.Lq ? __ldg(reinterpret_cast<const uint4*>(base + (long long)row * p.q_st) + c)
                                : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
          const uint32_t w[4] = {v[gi][i].x, v[gi][i].y, v[gi][i].z, v[gi][i].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] += __uint_as_float(w[e] << 16);
            acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) sum[e] += acc[e];
      }
    }
    const int nrows = min(64, p.Lq - qb * 64);
#pragma unroll
    for (int e = 0; e < 8; ++e) qs[q * D + c * 8 + e] = sum[e] * (1.f / (float)nrows);
  }
}

// Ranking keys of the n_win_blk window blocks for the nq pooled query blocks:
// thread st scores blocks st, st + 64, ... from the block means in global memory
// (four multiply-add chains over the float4 columns, two of them per paired
// f32x2 operation, added pairwise at the end).
template <int D>
__device__ __forceinline__ void fs_score(const AttnParams& p, int s, int nq, const float* qs, uint32_t* keys,
                                         int st) {
  constexpr int CH = D / 4;
  const float* kb = p.kbar + (size_t)s * p.n_win_blk * D;
  const float4* q4 = reinterpret_cast<const float4*>(qs);
  for (int w = st; w < p.n_win_blk; w += 64) {
    const float4* kr = reinterpret_cast<const float4*>(kb + (size_t)w * D);
    uint64_t acc[4][2];  // per query block: chains (x, y) and (z, w)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = 0ull;
#pragma unroll 8
    for (int cc = 0; cc < CH; ++cc) {
      const float4 kv = __ldg(kr + cc);
      const uint64_t k01 = pack2f(kv.x, kv.y), k23 = pack2f(kv.z, kv.w);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 qv = q4[q * CH + cc];
        acc[q][0] = fma2f(pack2f(qv.x, qv.y), k01, acc[q][0]);
        acc[q][1] = fma2f(pack2f(qv.z, qv.w), k23, acc[q][1]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float a0, a1, a2, a3;
      unpack2f(acc[q][0], a0, a1);
      unpack2f(acc[q][1], a2, a3);
      if (q < nq) keys[q * p.n_win_blk + w] = score_key(rank_score((a0 + a1) + (a2 + a3)));
    }
  }
}

// 32 fp32 values -> 32 bf16 at dst (64 bytes, 16-byte aligned).
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const float* v) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = w;
  }
}

__device__ __forceinline__ void load_row32(const __nv_bfloat16* src, float* v) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 w = s4[q];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * q + 2 * e + 0] = __uint_as_float(ws[e] << 16);
      v[8 * q + 2 * e + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
    }
  }
}

// 32 fp32 values v -> at dst, bf16 of v - float(bf16(v)) (what rounding v to bf16
// drops; v = bf16(v) + residual to within 2^-17 |v|).
__device__ __forceinline__ void store_residual32(__nv_bfloat16* dst, const float* v) {
  float r[32];
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const uint32_t h = pack_bf16x2(v[e], v[e + 1]);
    r[e] = v[e] - __uint_as_float(h << 16);
    r[e + 1] = v[e + 1] - __uint_as_float(h & 0xFFFF0000u);
  }
  store_row32(dst, r);
}

// 32 values rebuilt as bf16 row + bf16 residual row (see store_residual32).
__device__ __forceinline__ void load_residual32(const __nv_bfloat16* row, const __nv_bfloat16* res, float* v) {
  float a[32], b[32];
  load_row32(row, a);
  load_row32(res, b);
#pragma unroll
  for (int e = 0; e < 32; ++e) v[e] = a[e] + b[e];
}

// 32 fp32 values stored as two bf16-sized rows: the high 16 bits of each value
// at `hi`, the low 16 bits at `lo` (64 bytes each, 16-byte aligned).
__device__ __forceinline__ void store_split32(__nv_bfloat16* hi, __nv_bfloat16* lo, const uint32_t* v) {
  uint4* h4 = reinterpret_cast<uint4*>(hi);
  uint4* l4 = reinterpret_cast<uint4*>(lo);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t a = v[8 * q + 2 * e], b = v[8 * q + 2 * e + 1];
      hw[e] = (b & 0xFFFF0000u) | (a >> 16);
      lw[e] = (b << 16) | (a & 0xFFFFu);
    }
    h4[q] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    l4[q] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

__device__ __forceinline__ void load_split32(const __nv_bfloat16* hi, const __nv_bfloat16* lo, float* v) {
  const uint4* h4 = reinterpret_cast<const uint4*>(hi);
  const uint4* l4 = reinterpret_cast<const uint4*>(lo);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 H = h4[q], L = l4[q];
    const uint32_t hw[4] = {H.x, H.y, H.z, H.w}, lw[4] = {L.x, L.y, L.z, L.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * q + 2 * e] = __uint_as_float((hw[e] << 16) | (lw[e] & 0xFFFFu));
      v[8 * q + 2 * e + 1] = __uint_as_float((hw[e] & 0xFFFF0000u) | (lw[e] >> 16));
    }
  }
}

// exp2 on the FMA pipe for kExpEmu16 of every 16 score columns, which takes that
// share of the exponentials off the MUFU pipe (one exponential per score).
// 2^x = 2^r * q(f): r = round(x) by the 1.5 * 2^23 rounding trick, f = x - r in
// [-1/2, 1/2], q the cubic that minimises the maximum relative error of q(f) / 2^f
// on that interval (Lawson's iteratively reweighted least squares, fp32
// coefficients; fit_exp2_poly.py beside this file reproduces them): max relative
// error 7.5e-5, far below the 2^-9 rounding of P to bf16.  2^r is added into the
// exponent field as an integer.  Arguments are clamped to -126 first, so -inf
// (a masked score) gives at most 2^-126, which no output can resolve.
#ifndef VKV_EXP_EMU16
#define VKV_EXP_EMU16 4
#endif
constexpr int kExpEmu16 = VKV_EXP_EMU16;

// The fused merge keeps the earlier branch's partial as its final bf16 row plus a
// bf16 residual row (1), or as an exact high/low 16-bit split rewritten at the end (0).
#ifndef VKV_MERGE_RESIDUAL
#define VKV_MERGE_RESIDUAL 1
#endif

// L2 prefetch of the earlier branch's split rows before the final epilogue (1 = on).
#ifndef VKV_EPI_PREFETCH
#define VKV_EPI_PREFETCH 1
#endif


// Development timeline (compiled only with -DVKV_TRACE): SM clock stamps of the
// pipeline events of CTA 0, read back with vkv_debug_trace().
#ifdef VKV_TRACE
__device__ unsigned long long g_vkv_trace[2 * 28672];
#define VKV_STAMP(idx)                                                        \
  do {                                                                        \
    const int i_ = (idx);                                                     \
    if (blockIdx.x == 0 && i_ >= 0 && i_ < 28672) {                           \
      g_vkv_trace[i_] = clock64();                                            \
      g_vkv_trace[28672 + i_] = globaltimer();                                \
    }                                                                         \
  } while (0)
#else
#define VKV_STAMP(idx) \
  do {                 \
  } while (0)
#endif
// 2^x for a pair of arguments (x <= 8).  Arguments below -126 give a value of
// at most 2^-126 (masked scores are -inf), which no output can resolve.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& e0, float& e1) {
  const uint64_t xc = pack2f(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t magic = pack2f(12582912.f, 12582912.f);
  const uint64_t t = add2f(xc, magic);
  const uint64_t f = sub2f(xc, sub2f(t, magic));
  uint64_t q = fma2f(pack2f(0.0551716685f, 0.0551716685f), f, pack2f(0.242611140f, 0.242611140f));
  q = fma2f(q, f, pack2f(0.693260968f, 0.693260968f));
  q = fma2f(q, f, pack2f(0.999928057f, 0.999928057f));
  float q0, q1, t0, t1;
  unpack2f(q, q0, q1);
  unpack2f(t, t0, t1);
  e0 = __uint_as_float(__float_as_uint(t0) * 8388608u + __float_as_uint(q0));
  e1 = __uint_as_float(__float_as_uint(t1) * 8388608u + __float_as_uint(q1));
}

constexpr float kLn2 = 0.6931471805599453f;

// Output branches of a launch: SEGMENTS has n_branches, the other modes one.
__device__ __forceinline__ int out_branches(const AttnParams& p) {
  return p.mode == VKV_MODE_SEGMENTS ? p.n_branches : 1;
}

// Key-axis pieces.  A piece of a split unit leaves, per branch it reached, O / l
// (fp32) and its LSE (natural log) in its workspace slot; the combine kernel,
// launched behind the attention grid, merges a unit's pieces (the LSE merge,
// the same as between branches).  Slot rows: [slot][tile 2][branch nbr][row 128].
__device__ __forceinline__ size_t piece_row_n(int nbr, int slot, int t, int br, int r) {
  return ((size_t)(slot * 2 + t) * nbr + br) * 128 + r;
}
__device__ __forceinline__ size_t piece_row(const AttnParams& p, int slot, int t, int br, int r) {
  return piece_row_n(out_branches(p), slot, t, br, r);
}

// Workspace slot of piece entry k.
__device__ __forceinline__ int piece_slot(const AttnParams& p, int k) {
  const uint32_t y = p.pieces[k].y;
  return (int)(y & 0xFFFFu) + (int)((y >> 16) & 0xFFu);
}

// A piece's slot row holds a branch's exact fp32 partial O / l (D floats at
// ws_o) and its LSE (natural log, at ws_l).  The host fills ws_l with NaN before
// the launch, so a branch a piece did not reach reads as absent.

// A piece closes a branch into its workspace slot row (out of line, so that
// the softmax step loop keeps the register allocation of a whole unit).
template <int D>
__device__ __noinline__ void piece_close_branch(const AttnParams& p, int slot, int t, int br, int r, bool row_ok,
                                                uint32_t tO, float m, float l) {
  const size_t wrow = piece_row(p, slot, t, br, r);
  float* dst = p.ws_o + wrow * D;
  const bool has = l > 0.f;
  const float inv = has ? 1.f / l : 0.f;
#pragma unroll
  for (int c0 = 0; c0 < D; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tO + c0, v);
    tmem_ld_wait();
    reg_fence<32>(v);
    if (row_ok) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(dst + c0)[q] =
            make_float4(__uint_as_float(v[4 * q]) * inv, __uint_as_float(v[4 * q + 1]) * inv,
                        __uint_as_float(v[4 * q + 2]) * inv, __uint_as_float(v[4 * q + 3]) * inv);
    }
  }
  if (row_ok) p.ws_l[wrow] = has ? (m + lg2_approx(l)) * kLn2 : -INFINITY;
}

// Merges the pieces of the split units of one launch (one thread per 8 columns of
// a query row), after the attention grid before it on the stream has completed:
// per branch L = log sum_i e^L_i and O = sum_i e^(L_i - L) O_i, then the outputs as
// an unsplit unit writes them (branch rows, LSEs, and the merge of two branches).
// Launched as a programmatic dependent, so its blocks are placed while the
// attention grid drains.
template <int D>
__global__ void __launch_bounds__(256) piece_combine_kernel(const __grid_constant__ CombineParams c) {
  constexpr int TPR = D / 8;       // threads per row
  constexpr int RPB = 256 / TPR;   // rows per block
  constexpr int BPT = 128 / RPB;   // blocks per 128-row query tile
  constexpr float kLog2e = 1.4426950408889634f;
  griddep_wait();
  const int ui = blockIdx.x / (2 * BPT);
  const int t = (blockIdx.x / BPT) & 1;
  const int r = (blockIdx.x % BPT) * RPB + (int)threadIdx.x / TPR;
  const int c0 = ((int)threadIdx.x % TPR) * 8;
  if (ui >= c.n_units) return;
  const uint32_t code = c.code[ui];
  const int tile0 = (int)(code & 0xFFFu);
  const int ntiles = ((code >> 13) & 1u) ? 2 : 1;
  const int s = (int)(code >> 14);
  if (t >= ntiles) return;
  const int b = s / c.H, h = s - b * c.H;
  int qrow = (tile0 + t) * 128 + r;
  if (c.mode == VKV_MODE_BLOCK_SPARSE) {
    // the unit's query blocks follow qblk_order (the attention kernel reports a bad entry)
    const int pos = 2 * (tile0 + t) + (r >> 6);
    int qb = pos < c.n_qblk ? pos : -1;
    if (qb >= 0 && c.qblk_order) {
      const int q = __ldg(c.qblk_order + (size_t)s * c.n_qblk + pos);
      if (q >= 0 && q < c.n_qblk) qb = q;
    }
    qrow = qb >= 0 ? qb * 64 + (r & 63) : c.Lq;
  }
  if (qrow >= c.Lq) return;
  const int slot0 = (int)(c.slots[ui] & 0xFFFFu);
  const int n = (int)(c.slots[ui] >> 16);
  const bool do_merge = c.om != nullptr && c.nbr == 2;
  float L[2] = {-INFINITY, -INFINITY};
  float f[2][8];
#pragma unroll
  for (int br = 0; br < 2; ++br) {
#pragma unroll
    for (int e = 0; e < 8; ++e) f[br][e] = 0.f;
    if (br >= c.nbr) continue;
    float w[kMaxPiecesPerUnit];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kMaxPiecesPerUnit; ++i) {
      float x = -INFINITY;
      if (i < n) {
        x = __ldcg(c.ws_l + piece_row_n(c.nbr, slot0 + i, t, br, r));
        x = (x == x) ? x * kLog2e : -INFINITY;  // NaN: a branch this piece did not reach
      }
      w[i] = x;
      mx = fmaxf(mx, x);
    }
    float den = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPiecesPerUnit; ++i) {
      w[i] = (w[i] == -INFINITY) ? 0.f : ex2_approx(w[i] - mx);
      den += w[i];
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    L[br] = den > 0.f ? mx + lg2_approx(den) : -INFINITY;
#pragma unroll
    for (int i = 0; i < kMaxPiecesPerUnit; ++i) {
      if (w[i] > 0.f) {
        const float wi = w[i] * inv;
        const float4* src = reinterpret_cast<const float4*>(c.ws_o + piece_row_n(c.nbr, slot0 + i, t, br, r) * D + c0);
        const float4 A = __ldcg(src), B2 = __ldcg(src + 1);
        f[br][0] = fmaf(wi, A.x, f[br][0]);
        f[br][1] = fmaf(wi, A.y, f[br][1]);
        f[br][2] = fmaf(wi, A.z, f[br][2]);
        f[br][3] = fmaf(wi, A.w, f[br][3]);
        f[br][4] = fmaf(wi, B2.x, f[br][4]);
        f[br][5] = fmaf(wi, B2.y, f[br][5]);
        f[br][6] = fmaf(wi, B2.z, f[br][6]);
        f[br][7] = fmaf(wi, B2.w, f[br][7]);
      }
    }
    __nv_bfloat16* orow = c.o[br] + b * c.o_sb[br] + (long long)qrow * c.o_st[br] + h * c.o_sh[br] + c0;
    *reinterpret_cast<uint4*>(orow) = make_uint4(pack_bf16x2(f[br][0], f[br][1]), pack_bf16x2(f[br][2], f[br][3]),
                                                 pack_bf16x2(f[br][4], f[br][5]), pack_bf16x2(f[br][6], f[br][7]));
    if (c0 == 0) c.lse[br][(size_t)s * c.Lq + qrow] = (L[br] == -INFINITY) ? -INFINITY : L[br] * kLn2;
  }
  if (do_merge) {
    const float M = fmaxf(L[0], L[1]);
    const float Ms = (M == -INFINITY) ? 0.f : M;
    const float e0 = (L[0] == -INFINITY) ? 0.f : ex2_approx(L[0] - Ms);
    const float e1 = (L[1] == -INFINITY) ? 0.f : ex2_approx(L[1] - Ms);
    const float den = e0 + e1;
    const float a0 = den > 0.f ? e0 / den : 0.f, a1 = den > 0.f ? e1 / den : 0.f;
    float g[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) g[e] = fmaf(a0, f[0][e], a1 * f[1][e]);
    __nv_bfloat16* mrow = c.om + b * c.om_sb + (long long)qrow * c.om_st + h * c.om_sh + c0;
    *reinterpret_cast<uint4*>(mrow) = make_uint4(pack_bf16x2(g[0], g[1]), pack_bf16x2(g[2], g[3]),
                                                 pack_bf16x2(g[4], g[5]), pack_bf16x2(g[6], g[7]));
    if (c0 == 0) c.lsem[(size_t)s * c.Lq + qrow] = (M == -INFINITY) ? -INFINITY : (Ms + lg2_approx(den)) * kLn2;
  }
}

// Register split between the producer/MMA warpgroup and the two softmax
// warpgroups.  setmaxnreg.inc only succeeds if the total stays within what the
// CTA was launched with (384 threads x 168 registers); the host checks the
// compiled register count against kRegsLaunchNeeded before every launch.
constexpr int kRegsProducer = 88;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsLaunchNeeded = (128 * kRegsProducer + 256 * kRegsSoftmax + 383) / 384;
static_assert(128 * kRegsProducer + 256 * kRegsSoftmax <= 384 * 168, "register split");
constexpr float kRescaleThreshold = 8.0f;  // log2 units

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xFFFFFFFFu, v); }

// SP: the block-sparse instantiation.  It keeps two block lists, so the next
// unit's list and its first copies are ready before the current unit ends; the
// second list lives in the last K/V slot, which its ring then leaves out.
// PC: the schedule has key-axis pieces.  Kept apart because the piece paths,
// though cold, change the register allocation of the softmax step loop (measured
// ~10 % more cycles per step on whole units with them compiled in).
// FS (with SP, without PC): warps 2-3 select each unit's window blocks from the
// cached window block means; the other roles read the unit's block list in two
// steps (the persistent prefix, then the rest once the selection is done).
template <int D, bool SP, bool PC, bool FS = false>
__global__ void __launch_bounds__(384, 1) chunk_attn_kernel(const __grid_constant__ AttnParams p) {
  static_assert(!FS || (SP && !PC), "selection in the kernel: block-sparse, whole units");
  using C = AttnCfg<D>;
  constexpr uint32_t NS = SP ? (uint32_t)C::NSLOT - 1u : (uint32_t)C::NSLOT;  // ring slots
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::OFF_CTL);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sKV = sbase + C::OFF_KV;
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  volatile int* abort_flag = &ctl->abort_flag;
  const uint32_t b_full0 = smem_u32(&ctl->full[0]);
  const uint32_t b_empty0 = smem_u32(&ctl->empty[0]);
  const uint32_t b_qfull = smem_u32(&ctl->q_full);
  const uint32_t b_qempty = smem_u32(&ctl->q_empty);
  const uint32_t b_sfull0 = smem_u32(&ctl->s_full[0]);
  const uint32_t b_pfull0 = smem_u32(&ctl->p_full[0]);
  const uint32_t b_odone0 = smem_u32(&ctl->o_done[0]);
  const uint32_t b_lready0 = smem_u32(&ctl->list_ready[0]);
  const uint32_t b_lfree0 = smem_u32(&ctl->list_free[0]);
  const uint32_t b_lpers0 = smem_u32(&ctl->list_pers[0]);
  const uint32_t b_drain = smem_u32(&ctl->drain);
  const uint32_t b_kx = smem_u32(&ctl->kx_sync);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(b_full0 + 8 * i, 1);
      mbar_init(b_empty0 + 8 * i, 1);
    }
    mbar_init(b_qfull, 1);
    mbar_init(b_qempty, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(b_sfull0 + 8 * t, 1);
      mbar_init(b_pfull0 + 8 * t, 4);
      mbar_init(b_odone0 + 8 * t, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_lready0 + 8 * b, 1);
      // readers of a list buffer: the MMA thread, the 8 softmax warps, and in the
      // block-sparse instantiation (whose lists warps 2-3 build) the producer
      mbar_init(b_lfree0 + 8 * b, SP ? 10 : 9);
      mbar_init(b_lpers0 + 8 * b, 1);
    }
    mbar_init(b_drain, 1);
    if (FS) mbar_init(smem_u32(&ctl->kx_sync), 8);
    ctl->abort_flag = 0;
    ctl->list_count[0] = 0;
    ctl->list_count[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the piece combine kernel behind this grid may be placed as SMs free up; it waits
  // for this whole grid before it reads a partial
  if (PC) griddep_launch_dependents();
  const uint32_t tmem = ctl->tmem_base;
  const int u_begin = p.cta_begin[blockIdx.x];
  const int u_end = p.cta_begin[blockIdx.x + 1];
  const bool sparse = p.mode == VKV_MODE_BLOCK_SPARSE;
  const bool ragged = p.mode == VKV_MODE_RAGGED;
  uint32_t* const list1 = reinterpret_cast<uint32_t*>(smem + C::OFF_KV + (C::NSLOT - 1) * C::KV_BYTES);
  auto list_buf = [&](int b) { return (SP && b) ? list1 : ctl->list; };

  if (warp < 4) {
    setmaxnreg_dec<kRegsProducer>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      uint32_t item = 0, qcnt = 0, ucnt = 0;
      int piece_k = p.cta_piece0[blockIdx.x];
      bool ok = true;
      for (int ui = u_begin; ui < u_end; ++ui, ++ucnt) {
        const UnitInfo u = decode_entry<PC>(p, p.units[ui]);
        int rs = 0, rl = 0;
        const int lb = SP ? (int)(ucnt & 1u) : 0;
        const uint32_t uph = (ucnt >> 1) & 1u;  // FS: this list buffer's use parity
        bool fs_full = true;                     // FS: the whole block list is known
        if (FS) {
          // the selection warps build the list: start on its persistent prefix
          bool w = true;
          if (lane == 0) w = mbar_wait(b_lpers0 + 8 * lb, uph, abort_flag, p.err);
          ok = __shfl_sync(0xFFFFFFFFu, w ? 1 : 0, 0) != 0;
          if (!ok) break;
          if ((ctl->pers_count[lb] >> 1) == 0) {
            if (lane == 0) w = mbar_wait(b_lready0 + 8 * lb, uph, abort_flag, p.err);
            ok = __shfl_sync(0xFFFFFFFFu, w ? 1 : 0, 0) != 0;
            if (!ok) break;
          } else {
            fs_full = false;
          }
        } else if (SP) {
          // warp 2 builds the list
          bool w = true;
          if (lane == 0) w = mbar_wait(b_lready0 + 8 * lb, uph, abort_flag, p.err);
          ok = __shfl_sync(0xFFFFFFFFu, w ? 1 : 0, 0) != 0;
          if (!ok) break;
        } else if (sparse) {
          // wait for the unit that used this list buffer before (one unit back with a
          // single buffer, two with two) to release it
          const uint32_t back = SP ? 2u : 1u;
          if (ucnt >= back) {
            bool w = true;
            if (lane == 0) w = mbar_wait(b_lfree0 + 8 * lb, ((ucnt - back) / back) & 1, abort_flag, p.err);
            ok = __shfl_sync(0xFFFFFFFFu, w ? 1 : 0, 0) != 0;
            if (!ok) break;
          }
          build_block_list(p, ctl, u, list_buf(lb), &ctl->list_count[lb]);
          if (lane == 0) mbar_arrive(b_lready0 + 8 * lb);
        } else if (ragged) {
          ragged_range(p, u.s, rs, rl, lane == 0);
        }
        PieceInfo pi;
        int nsteps;
        if (FS) {
          pi.j0 = 0;
          nsteps = fs_full ? unit_steps(p, ctl->list_count[lb], 0) : (ctl->pers_count[lb] >> 1);
        } else {
          nsteps = entry_steps(p, u, unit_steps(p, ctl->list_count[lb], rl), piece_k, pi);
        }
        if (nsteps == 0) {
          if (SP && lane == 0) mbar_arrive(b_lfree0 + 8 * lb);
          continue;
        }
        if (lane == 0) {
          if (qcnt > 0) ok = mbar_wait(b_qempty, (qcnt - 1) & 1, abort_flag, p.err);
          if (ok) {
            mbar_arrive_expect_tx(b_qfull, (uint32_t)(u.ntiles * C::QT_BYTES));
            for (int t = 0; t < u.ntiles; ++t) {
              if (sparse) {
                // two 64-row query blocks in unit order; a missing one reads rows past
                // Lq, which the TMA fills with zeros
                for (int half = 0; half < 2; ++half) {
                  const int qb = unit_qblk(p, u.s, 2 * (u.tile0 + t) + half, false);
                  const int row = qb >= 0 ? qb * 64 : p.n_qblk * 64;
#pragma unroll
                  for (int ac = 0; ac < C::NAC; ++ac)
                    tma_load_4d(sQ + t * C::QT_BYTES + ac * C::ATOM + half * 64 * 128, &p.tm_q, ac * 64, u.h,
                                row, u.b, b_qfull);
                }
              } else {
#pragma unroll
                for (int ac = 0; ac < C::NAC; ++ac)
                  tma_load_4d(sQ + t * C::QT_BYTES + ac * C::ATOM, &p.tm_q, ac * 64, u.h,
                              (u.tile0 + t) * 128, u.b, b_qfull);
              }
            }
            ++qcnt;
          }
          TileIter it;
          it.init(&p, list_buf(lb), (FS && !fs_full) ? ctl->pers_count[lb] : ctl->list_count[lb], rs, rl);
          if (u.piece) it.seek(pi.j0);
          const int kvh = ragged ? 0 : u.h;
          const int kvb = ragged ? 0 : u.b;
          for (int j = 0; (FS || j < nsteps) && ok; ++j) {
            if (FS && j >= nsteps) {
              // end of the persistent prefix: the rest of the list once the selection is in
              if (fs_full) break;
              ok = mbar_wait(b_lready0 + 8 * lb, uph, abort_flag, p.err);
              if (!ok) break;
              fs_full = true;
              it.count = ctl->list_count[lb];
              nsteps = unit_steps(p, it.count, 0);
              if (j >= nsteps) break;
            }
            const TileDesc td = it.next();
            for (int kv = 0; kv < 2; ++kv) {
              const uint32_t slot = item % NS, use = item / NS;
              if (use > 0) ok = mbar_wait(b_empty0 + 8 * slot, (use - 1) & 1, abort_flag, p.err);
              if (!ok) break;
#ifdef VKV_TEST_AIDS
              if (item == 0 && p.withhold_first_copy) {
                ++item;  // test aid: this copy never arrives, so the wait for it runs out
                continue;
              }
#endif
              VKV_STAMP(20480 + (int)item);
              mbar_arrive_expect_tx(b_full0 + 8 * slot, (uint32_t)C::KV_BYTES);
              const CUtensorMap* tm = kv ? &p.tm_v : &p.tm_k;
              const uint32_t dst = sKV + slot * C::KV_BYTES;
#pragma unroll
              for (int ac = 0; ac < C::NAC; ++ac) {
                tma_load_4d(dst + ac * C::ATOM, tm, ac * 64, kvh, td.rowA, kvb, b_full0 + 8 * slot);
                tma_load_4d(dst + ac * C::ATOM + 64 * 128, tm, ac * 64, kvh, td.rowB, kvb,
                            b_full0 + 8 * slot);
              }
              ++item;
            }
          }
          if (SP && ok) mbar_arrive(b_lfree0 + 8 * lb);  // this unit's list entries are all read
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      if (!ok && lane == 0) {
        // let copies already issued land before the CTA exits
        for (uint32_t i = (item > NS ? item - NS : 0); i < item; ++i)
          mbar_wait_drain(b_full0 + 8 * (i % NS), (i / NS) & 1);
        if (qcnt > 0) mbar_wait_drain(b_qfull, (qcnt - 1) & 1);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      // Per step j and tile t: O_t += P_t(j) V_j (A = P_t from TMEM), then
      // S_t(j+1) = Q_t K_{j+1}^T; each after a suspending wait on its inputs.
      if (lane == 0) {
        constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);
        uint32_t item = 0, qcnt = 0, ucnt = 0;
        uint32_t pv_cnt[2] = {0, 0};  // PV products issued on accumulator t
        uint32_t pv_par = 0;          // FS: bit t = parity of pv_cnt[t] (t varies per step there)
        int piece_k = p.cta_piece0[blockIdx.x];
        bool ok = true;
        auto wait_item = [&](uint32_t it_) {
          return mbar_wait(b_full0 + 8 * (it_ % NS), (it_ / NS) & 1, abort_flag, p.err);
        };
        auto issue_qk = [&](int t, uint32_t kslot, int qt) {
          const uint32_t d_tm = tmem + (uint32_t)(t * 128);
          const uint32_t qa = sQ + qt * C::QT_BYTES;
          const uint32_t kb = sKV + kslot * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::ATOM + (kk & 3) * 32;
            mma_bf16_ss(d_tm, sdesc_k_sw128(qa + off), sdesc_k_sw128(kb + off), IDESC_QK, kk > 0);
          }
          mma_commit(b_sfull0 + 8 * t);
        };
        for (int ui = u_begin; ui < u_end && ok; ++ui, ++ucnt) {
          const UnitInfo u = decode_entry<PC>(p, p.units[ui]);
          const bool kx = FS && p.kx && u.ntiles == 1;
          int rs = 0, rl = 0;
          const int lb = SP ? (int)(ucnt & 1u) : 0;
          const uint32_t uph = SP ? ((ucnt >> 1) & 1u) : (ucnt & 1u);  // this buffer's use parity
          if (sparse) {
            ok = mbar_wait((FS ? b_lpers0 : b_lready0) + 8 * lb, uph, abort_flag, p.err);
            if (!ok) break;
          } else if (ragged) {
            ragged_range(p, u.s, rs, rl, false);
          }
          PieceInfo pi;
          int nsteps;
          bool fs_full = true;  // FS: the unit's step count is final
          if (FS) {
            // the persistent prefix alone fixes a lower bound; the count itself is
            // needed one step before the prefix ends (whether another S follows; two
            // steps before it when the steps alternate between the accumulators)
            pi.j0 = 0;
            nsteps = ctl->pers_count[lb] >> 1;
            if (nsteps <= (kx ? 2 : 1)) {
              ok = mbar_wait(b_lready0 + 8 * lb, uph, abort_flag, p.err);
              if (!ok) break;
              nsteps = unit_steps(p, ctl->list_count[lb], 0);
              mbar_arrive(b_lfree0 + 8 * lb);
            } else {
              fs_full = false;
            }
          } else {
            nsteps = entry_steps(p, u, unit_steps(p, ctl->list_count[lb], rl), piece_k, pi);
            if (sparse) mbar_arrive(b_lfree0 + 8 * lb);  // only the step count was needed
          }
          if (nsteps == 0) continue;
          TileIter it;
          it.init(&p, list_buf(lb), ctl->list_count[lb], rs, rl);
          if (u.piece) it.seek(pi.j0);
          ok = mbar_wait(b_qfull, qcnt & 1, abort_flag, p.err);
          ++qcnt;
          if (!ok) break;
          // prologue: S_t(0) = Q_t K_0^T.  A one-tile unit whose key steps alternate
          // between the accumulators (kx) computes S_(j&1) = Q K_j^T and
          // O_(j&1) += P_(j&1) V_j instead, so the two softmax warpgroups overlap as
          // on two tiles: its prologue is S_0 = Q K_0^T and S_1 = Q K_1^T, and each
          // S_t is next computed two steps later.
          const int kxi = kx ? 1 : 0;
          ok = wait_item(item);
          if (!ok) break;
          tc_fence_after();
          for (int t = 0; t < u.ntiles; ++t) issue_qk(t, item % NS, t);
          mma_commit(b_empty0 + 8 * (item % NS));
          if (kx && nsteps > 1) {
            ok = wait_item(item + 2);
            if (!ok) break;
            tc_fence_after();
            issue_qk(1, (item + 2) % NS, 0);
            mma_commit(b_empty0 + 8 * ((item + 2) % NS));
          }
          bool q_rel = kx ? nsteps <= 2 : nsteps == 1;  // the Q tiles' release is committed
          if (q_rel) mma_commit(b_qempty);
          for (int j = 0; j < nsteps && ok; ++j) {
            if (FS && !fs_full && j + 1 + kxi >= nsteps) {
              ok = mbar_wait(b_lready0 + 8 * lb, uph, abort_flag, p.err);
              if (!ok) break;
              nsteps = unit_steps(p, ctl->list_count[lb], 0);
              fs_full = true;
              mbar_arrive(b_lfree0 + 8 * lb);
            }
            // a piece may start inside a branch: its first step starts the accumulator too
            const bool first = (sparse || ragged) ? (kx ? j <= 1 : j == 0) : (it.next().first || (PC && j == 0));
            const uint32_t vit = item + 2 * j + 1;
            const uint32_t knext = item + 2 * j + 2 + 2 * kxi;
            const bool has_next = j + 1 + kxi < nsteps;
            const int trm = (pv_cnt[0] < 256) ? 16384 + (int)(pv_cnt[0]) * 16 : -100;
            ok = wait_item(vit);
            if (!ok) break;
            VKV_STAMP(trm);
            bool k_ready = false;
            const int t_end = kx ? (j & 1) + 1 : u.ntiles;
            for (int t = kx ? (j & 1) : 0; t < t_end && ok; ++t) {
              ok = mbar_wait(b_pfull0 + 8 * t, FS ? ((pv_par >> t) & 1u) : (pv_cnt[t] & 1u), abort_flag, p.err);
              if (!ok) break;
              VKV_STAMP(trm + 1 + 4 * t);
              tc_fence_after();
              {
                const uint32_t d_tm = tmem + C::TM_O + (uint32_t)(t * D);
                const uint32_t pa = tmem + (uint32_t)(t * 128);
                const uint32_t vb = sKV + (vit % NS) * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  mma_bf16_ts(d_tm, pa + 8 * kk, sdesc_mn_sw128(vb + kk * 2048, C::ATOM), IDESC_PV,
                              (!first || kk > 0) ? 1u : 0u);
              }
              mma_commit(b_odone0 + 8 * t);
              VKV_STAMP(trm + 2 + 4 * t);
              if (FS)
                pv_par ^= 1u << t;
              else
                ++pv_cnt[t];
              if (has_next) {
                if (!k_ready) {
                  ok = wait_item(knext);
                  if (!ok) break;
                  tc_fence_after();
                  k_ready = true;
                  VKV_STAMP(trm + 3 + 4 * t);
                }
                issue_qk(t, knext % NS, kx ? 0 : t);
                VKV_STAMP(trm + 4 + 4 * t);
              }
            }
            if (!ok) break;
            mma_commit(b_empty0 + 8 * (vit % NS));
            if (has_next) {
              mma_commit(b_empty0 + 8 * (knext % NS));
              if (j + 2 + kxi == nsteps && fs_full) {
                mma_commit(b_qempty);
                q_rel = true;
              }
            } else if (FS && !q_rel) {
              // the count became final only at this last step: release the Q tiles now
              mma_commit(b_qempty);
              q_rel = true;
            }
          }
          item += 2 * nsteps;
        }
        // every MMA issued so far completes before TMEM is released
        mma_commit(b_drain);
        mbar_wait_drain(b_drain, 0);
      }
      __syncwarp();
    } else if (SP && !FS && warp == 2) {
      // ------------------------------------------------------------ block lists (warp 2)
      // Each unit's block list from the caller's selection, up to one unit ahead of the
      // other roles (the list buffer of unit i is free once every reader has finished
      // unit i - 2), so the producer only waits for it.
      uint32_t ucnt = 0;
      for (int ui = u_begin; ui < u_end; ++ui, ++ucnt) {
        const UnitInfo u = decode_entry<PC>(p, p.units[ui]);
        const int lb = (int)(ucnt & 1u);
        if (ucnt >= 2) {
          bool w = true;
          if (lane == 0) w = mbar_wait(b_lfree0 + 8 * lb, ((ucnt - 2) >> 1) & 1u, abort_flag, p.err);
          if (__shfl_sync(0xFFFFFFFFu, w ? 1 : 0, 0) == 0) break;
        }
        build_block_list(p, ctl, u, list_buf(lb), &ctl->list_count[lb]);
        if (lane == 0) mbar_arrive(b_lready0 + 8 * lb);
      }
    } else if (FS) {
      // ------------------------------------------------------------ selection (warps 2-3)
      // Runs up to one unit ahead of the other roles: the list buffer of unit i
      // is free once every reader has finished unit i - 2.
      const int st = (int)threadIdx.x - 64;
      const int sw = warp - 2;
      uint8_t* const scr = reinterpret_cast<uint8_t*>(list1);
      float* const qs = reinterpret_cast<float*>(scr + FsScratch<D>::OFF_QS);
      int* const hist = reinterpret_cast<int*>(scr + FsScratch<D>::OFF_HIST);
      uint32_t* const keys = reinterpret_cast<uint32_t*>(scr + FsScratch<D>::OFF_KEYS);
      uint32_t ucnt = 0;
      for (int ui = u_begin; ui < u_end; ++ui, ++ucnt) {
        const UnitInfo u = decode_entry<false>(p, p.units[ui]);
        const int lb = (int)(ucnt & 1u);
        if (ucnt >= 2) {
          // one thread waits; both warps take its answer, so they never part ways
          if (st == 0)
            ctl->sel_go = mbar_wait(b_lfree0 + 8 * lb, ((ucnt - 2) >> 1) & 1u, abort_flag, p.err) ? 1 : 0;
          fs_bar();
          if (!ctl->sel_go) break;
        }
        const int qb0 = u.tile0 * 2;
        const int nqb = min(2 * u.ntiles, p.n_qblk - qb0);
        uint32_t* const list = list_buf(lb);
        if (sw == 0) {
          const int base = build_persist_prefix(p, u.s, nqb, list);
          if (lane == 0) ctl->pers_count[lb] = base;
          __threadfence_block();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_lpers0 + 8 * lb);
        }
        fs_pool<D>(p, u, qb0, nqb, qs, st);
        fs_bar();
        fs_score<D>(p, u.s, nqb, qs, keys, st);
        fs_bar();
        for (int q = sw; q < nqb; q += 2) {
          const int qbi = unit_qblk(p, u.s, qb0 + q, false);
          warp_topk(keys + q * p.n_win_blk, p.n_win_blk, p.topk, hist + sw * 256,
                    p.sel_out ? p.sel_out + ((size_t)u.s * p.n_qblk + qbi) * p.topk : nullptr, ctl->bitmap[q]);
        }
        fs_bar();
        if (sw == 0) {
          build_window_union(p, ctl, nqb, list, ctl->pers_count[lb], &ctl->list_count[lb]);
          if (lane == 0) mbar_arrive(b_lready0 + 8 * lb);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax
    setmaxnreg_inc<kRegsSoftmax>();
    const int t = (warp >= 8) ? 1 : 0;
    const int quarter = warp & 3;
    const int r = quarter * 32 + (int)lane;  // row inside the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + (uint32_t)(t * 128);
    const uint32_t tO = tmem + lane_base + C::TM_O + (uint32_t)(t * D);
    const uint32_t b_sfull = b_sfull0 + 8 * t;
    const uint32_t b_pfull = b_pfull0 + 8 * t, b_odone = b_odone0 + 8 * t;
    const float sl2 = p.scale_log2;
    uint32_t sf_cnt = 0, np = 0, ucnt = 0;
    int piece_k = p.cta_piece0[blockIdx.x];
    bool ok = true;
    for (int ui = u_begin; ui < u_end && ok; ++ui, ++ucnt) {
      const UnitInfo u = decode_entry<PC>(p, p.units[ui]);
      int rs = 0, rl = 0;
      const int lb = SP ? (int)(ucnt & 1u) : 0;
      const uint32_t uph = SP ? ((ucnt >> 1) & 1u) : (ucnt & 1u);
      if (sparse) {
        ok = warp_all(mbar_wait((FS ? b_lpers0 : b_lready0) + 8 * lb, uph, abort_flag, p.err));
        if (!ok) break;
      } else if (ragged) {
        ragged_range(p, u.s, rs, rl, false);
      }
      // a piece's details are re-read from the parameters where needed (its entry
      // is piece_k - 1), so that the step loop keeps no more state live than a
      // whole unit does
      PieceInfo pi0;
      int nsteps;
      bool fs_full = true;  // FS: the whole block list is known
      if (FS) {
        pi0.j0 = 0;
        nsteps = ctl->pers_count[lb] >> 1;
        if (nsteps == 0) {
          ok = warp_all(mbar_wait(b_lready0 + 8 * lb, uph, abort_flag, p.err));
          if (!ok) break;
          nsteps = unit_steps(p, ctl->list_count[lb], 0);
        } else {
          fs_full = false;
        }
      } else {
        nsteps = entry_steps(p, u, unit_steps(p, ctl->list_count[lb], rl), piece_k, pi0);
      }
      // a one-tile unit whose key steps alternate between the warpgroups: both
      // work on query tile 0, warpgroup t on the steps j with j % 2 == t
      const bool kx = FS && p.kx && u.ntiles == 1;
      const int tq = kx ? 0 : t;  // the query tile of this thread's row
      const bool active = kx || t < u.ntiles;
      int qrow = (u.tile0 + tq) * 128 + r;
      if (sparse) {
        const int qbr = unit_qblk(p, u.s, 2 * (u.tile0 + tq) + (r >> 6), false);
        qrow = qbr >= 0 ? qbr * 64 + (r & 63) : p.Lq;
      }
      const bool row_ok = qrow < p.Lq;
      const int qb = 2 * tq + (r >> 6);
      float m = -INFINITY, l = 0.f;            // running state of the current branch
      float m_prev = -INFINITY, l_prev = 0.f;  // state of the branch closed before it
      int cur_branch = -1, prev_branch = -1;
      if (active && nsteps > 0) {
        TileIter it;
        it.init(&p, list_buf(lb), (FS && !fs_full) ? ctl->pers_count[lb] : ctl->list_count[lb], rs, rl);
        if (u.piece) it.seek(pi0.j0);
        for (int j = 0; FS || j < nsteps; ++j) {
          if (FS && j >= nsteps) {
            // end of the persistent prefix: the rest of the list once the selection is in
            if (fs_full) break;
            ok = warp_all(mbar_wait(b_lready0 + 8 * lb, uph, abort_flag, p.err));
            if (!ok) break;
            fs_full = true;
            it.count = ctl->list_count[lb];
            nsteps = unit_steps(p, it.count, 0);
            if (j >= nsteps) break;
          }
          const TileDesc td = it.next();
          if (kx && (j & 1) != t) continue;  // the other warpgroup's step (its first is j = t)
          const int tr = (lane == 0 && sf_cnt < 128) ? t * 8192 + quarter * 2048 + (int)sf_cnt * 16 : -1;
          VKV_STAMP(tr);
          ok = warp_all(mbar_wait(b_sfull, sf_cnt & 1, abort_flag, p.err));
          VKV_STAMP(tr < 0 ? -1 : tr + 1);
          ++sf_cnt;
          if (!ok) break;
          tc_fence_after();
          uint32_t sr[128];
          tmem_ld32(tS + 0, sr + 0);
          tmem_ld32(tS + 32, sr + 32);
          tmem_ld32(tS + 64, sr + 64);
          tmem_ld32(tS + 96, sr + 96);
          tmem_ld_wait();
          reg_fence<128>(sr);
          VKV_STAMP(tr < 0 ? -1 : tr + 2);
          bool pending_epi = false;
          if (td.first || (PC && j == 0) || (kx && j == t)) {
            if (cur_branch >= 0) {
              pending_epi = true;
              prev_branch = cur_branch;
              m_prev = m;
              l_prev = l;
            }
            cur_branch = td.branch;
            m = -INFINITY;
            l = 0.f;
          }
          // visibility of this tile for this row
          const int limA = ((td.maskA >> qb) & 1u) ? td.limA : 0;
          const int limB = ((td.maskB >> qb) & 1u) ? td.limB : 0;
          if (__any_sync(0xFFFFFFFFu, (limA < 64) || (limB < 64))) {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              if (c >= limA) sr[c] = __float_as_uint(-INFINITY);
              if (c >= limB) sr[64 + c] = __float_as_uint(-INFINITY);
            }
          }
          float mx8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mx8[i] = max3f(__uint_as_float(sr[i]), __uint_as_float(sr[8 + i]),
                                                     __uint_as_float(sr[16 + i]));
#pragma unroll
          for (int c = 24; c < 120; c += 16) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              mx8[i] = max3f(mx8[i], __uint_as_float(sr[c + i]), __uint_as_float(sr[c + 8 + i]));
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) mx8[i] = fmaxf(mx8[i], __uint_as_float(sr[120 + i]));
          const float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]),
                                 fmaxf(mx8[6], mx8[7]));
          const float mt = mx * sl2;
          VKV_STAMP(tr < 0 ? -1 : tr + 6);
          float alpha = 1.f;
          bool rescale = false;
          if (m == -INFINITY) {
            m = mt;
          } else if (mt > m + kRescaleThreshold) {
            alpha = ex2_approx(m - mt);
            m = mt;
            rescale = true;
          }
          const float mu = (m == -INFINITY) ? 0.f : m;
          // p = 2^(s * scale * log2 e - m): pairs on the f32x2 path, kExpEmu16 of every
          // 16 columns on the FMA pipe, the rest on MUFU; P (bf16 pairs) -> the first
          // 64 TMEM columns of S_t, 32 columns at a time
          const uint64_t sl2x2 = pack2f(sl2, sl2), nmu2 = pack2f(-mu, -mu);
          uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pk[32];
#pragma unroll
            for (int g = 0; g < 64; g += 16) {
              const int c0 = h * 64 + g;
              float a[16], e[16];
#pragma unroll
              for (int i = 0; i < 16; i += 2)
                unpack2f(fma2f(pack2f(__uint_as_float(sr[c0 + i]), __uint_as_float(sr[c0 + i + 1])), sl2x2, nmu2),
                         a[i], a[i + 1]);
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                if (i >= 16 - kExpEmu16) {
                  exp2_poly2(a[i], a[i + 1], e[i], e[i + 1]);
                } else {
                  e[i] = ex2_approx(a[i]);
                  e[i + 1] = ex2_approx(a[i + 1]);
                }
              }
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                acc2[(i >> 1) & 3] = add2f(acc2[(i >> 1) & 3], pack2f(e[i], e[i + 1]));
                pk[(g + i) >> 1] = pack_bf16x2(e[i], e[i + 1]);
              }
            }
            tmem_st32(tS + (uint32_t)(h * 32), pk);
            VKV_STAMP(tr < 0 ? -1 : tr + 7 + h);
          }
          float sum_lo, sum_hi;
          unpack2f(add2f(add2f(acc2[0], acc2[1]), add2f(acc2[2], acc2[3])), sum_lo, sum_hi);
          l = l * alpha + (sum_lo + sum_hi);
          VKV_STAMP(tr < 0 ? -1 : tr + 3);
          // O_t already holds every PV up to step j-1: S_t(j) was committed after
          // O_t += P_t(j-1) V_{j-1}, and a commit covers all earlier MMAs.
          const bool need_o = pending_epi || __any_sync(0xFFFFFFFFu, rescale);
          VKV_STAMP(tr < 0 ? -1 : tr + 4);
          if (PC && pending_epi && u.piece) {
            piece_close_branch<D>(p, piece_slot(p, piece_k - 1), t, prev_branch, r, row_ok, tO, m_prev, l_prev);
          } else if (pending_epi) {
            // close the previous branch: O / l and LSE
            const bool has = l_prev > 0.f;
            const float inv = has ? 1.f / l_prev : 0.f;
            __nv_bfloat16* orow = p.o[prev_branch] + u.b * p.o_sb[prev_branch] +
                                  (long long)qrow * p.o_st[prev_branch] + u.h * p.o_sh[prev_branch];
            const bool split_prev = p.om != nullptr && p.n_branches == 2 && !sparse && !ragged;
            __nv_bfloat16* mrow_split =
                split_prev ? p.om + u.b * p.om_sb + (long long)qrow * p.om_st + u.h * p.om_sh : nullptr;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t v[32];
              tmem_ld32(tO + c0, v);
              tmem_ld_wait();
              reg_fence<32>(v);
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * inv);
              if (row_ok) {
                if (split_prev) {
#if VKV_MERGE_RESIDUAL
                  // this branch's row gets its final value (rounded to bf16); the merged row
                  // keeps what rounding dropped, so the merge at the end sees the fp32 partial
                  // to within 2^-17 of its size
                  store_row32(orow + c0, reinterpret_cast<const float*>(v));
                  store_residual32(mrow_split + c0, reinterpret_cast<const float*>(v));
#else
                  // keep the exact fp32 partial for the merge: high halves in the merged
                  // row, low halves in this branch's row; both rows are rewritten at the end
                  store_split32(mrow_split + c0, orow + c0, v);
#endif
                } else {
                  store_row32(orow + c0, reinterpret_cast<const float*>(v));
                }
              }
            }
            if (row_ok)
              p.lse[prev_branch][(size_t)u.s * p.Lq + qrow] =
                  has ? (m_prev + lg2_approx(l_prev)) * kLn2 : -INFINITY;
          } else if (need_o) {
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t v[32];
              tmem_ld32(tO + c0, v);
              tmem_ld_wait();
              reg_fence<32>(v);
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
              tmem_st32(tO + c0, v);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          VKV_STAMP(tr < 0 ? -1 : tr + 5);
          if (lane == 0) mbar_arrive(b_pfull);
          ++np;
        }
        if (VKV_EPI_PREFETCH && ok && !u.piece && p.om != nullptr && p.n_branches == 2 && !sparse && !ragged &&
            prev_branch >= 0 && row_ok) {
          // the earlier branch's partial (the two rows written at its close, long before
          // and likely out of L2) is read by the epilogue below: bring it into L2 while
          // the last PV product completes
          const __nv_bfloat16* mr = p.om + u.b * p.om_sb + (long long)qrow * p.om_st + u.h * p.om_sh;
          const __nv_bfloat16* pr = p.o[prev_branch] + u.b * p.o_sb[prev_branch] +
                                    (long long)qrow * p.o_st[prev_branch] + u.h * p.o_sh[prev_branch];
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 64) {
            prefetch_l2(mr + c0);
            prefetch_l2(pr + c0);
          }
        }
        // (with alternating steps, warpgroup 1 has none in a one-step unit)
        if (ok && (!kx || nsteps > t)) ok = warp_all(mbar_wait(b_odone, (np - 1) & 1, abort_flag, p.err));
        if (kx) {
          // merge the two warpgroups' states (the LSE merge of two key subsets):
          // each publishes its rows' (m, l); once both have, warpgroup t writes
          // columns [t D/2, (t+1) D/2) of each row from both accumulators; neither
          // leaves the unit (after which the MMA may overwrite its O) before both
          // have read.  Both take both barrier phases on every path.
          float* const kxs =
              reinterpret_cast<float*>(smem + C::OFF_KV + (C::NSLOT - 1) * C::KV_BYTES + KxScratch<D>::OFF);
          kxs[(2 * t) * 128 + r] = m;
          kxs[(2 * t + 1) * 128 + r] = l;
          __threadfence_block();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_kx);
          const bool ok_a = warp_all(mbar_wait(b_kx, 0, abort_flag, p.err));
          if (ok && ok_a) {
            tc_fence_after();
            const float m0 = kxs[r], l0 = kxs[128 + r], m1 = kxs[256 + r], l1 = kxs[384 + r];
            const bool h0 = l0 > 0.f, h1 = l1 > 0.f;
            const float mm = fmaxf(h0 ? m0 : -INFINITY, h1 ? m1 : -INFINITY);
            const float a0 = h0 ? ex2_approx(m0 - mm) : 0.f;
            const float a1 = h1 ? ex2_approx(m1 - mm) : 0.f;
            const float den = a0 * l0 + a1 * l1;
            const float inv = den > 0.f ? 1.f / den : 0.f;
            const float w0 = a0 * inv, w1 = a1 * inv;
            __nv_bfloat16* orow = p.o[0] + u.b * p.o_sb[0] + (long long)qrow * p.o_st[0] + u.h * p.o_sh[0];
            const uint32_t tO0 = tmem + lane_base + C::TM_O;
#pragma unroll
            for (int cc = 0; cc < D / 2; cc += 32) {
              const int c0 = t * (D / 2) + cc;
              uint32_t v0[32], v1[32];
              tmem_ld32(tO0 + (uint32_t)c0, v0);
              tmem_ld32(tO0 + (uint32_t)(D + c0), v1);
              tmem_ld_wait();
              reg_fence<32>(v0);
              reg_fence<32>(v1);
              float f[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                // an accumulator without keys for this row (or never written in this
                // unit) is left out, not multiplied by zero
                const float x = h0 ? w0 * __uint_as_float(v0[e]) : 0.f;
                f[e] = h1 ? fmaf(w1, __uint_as_float(v1[e]), x) : x;
              }
              if (row_ok) store_row32(orow + c0, f);
            }
            if (t == 0 && row_ok)
              p.lse[0][(size_t)u.s * p.Lq + qrow] = den > 0.f ? (mm + lg2_approx(den)) * kLn2 : -INFINITY;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(b_kx);
          const bool ok_b = warp_all(mbar_wait(b_kx, 1, abort_flag, p.err));
          ok = ok && ok_a && ok_b;
        } else if (ok && !u.piece) {
          tc_fence_after();
          // close the last branch, and merge with the one before it when asked
          const int lb = cur_branch;
          const bool has = l > 0.f;
          const float inv = has ? 1.f / l : 0.f;
          const bool do_merge = p.om != nullptr && p.n_branches == 2 && !sparse && !ragged;
          const bool has_prev = prev_branch >= 0 && l_prev > 0.f;
          const float L_last = has ? m + lg2_approx(l) : -INFINITY;
          const float L_prev = has_prev ? m_prev + lg2_approx(l_prev) : -INFINITY;
          const float M = fmaxf(L_last, L_prev);
          const float Ms = (M == -INFINITY) ? 0.f : M;
          const float w_last = has ? ex2_approx(L_last - Ms) : 0.f;
          const float w_prev = has_prev ? ex2_approx(L_prev - Ms) : 0.f;
          const float den = w_last + w_prev;
          const float c_last = den > 0.f ? w_last / den : 0.f;
          const float c_prev = den > 0.f ? w_prev / den : 0.f;
          __nv_bfloat16* orow =
              p.o[lb] + u.b * p.o_sb[lb] + (long long)qrow * p.o_st[lb] + u.h * p.o_sh[lb];
          __nv_bfloat16* mrow =
              do_merge ? p.om + u.b * p.om_sb + (long long)qrow * p.om_st + u.h * p.om_sh : nullptr;
          const __nv_bfloat16* prow =
              prev_branch >= 0 ? p.o[prev_branch] + u.b * p.o_sb[prev_branch] +
                                     (long long)qrow * p.o_st[prev_branch] + u.h * p.o_sh[prev_branch]
                               : nullptr;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tO + c0, v);
            tmem_ld_wait();
            reg_fence<32>(v);
            float f[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]) * inv;
            if (row_ok) {
              store_row32(orow + c0, f);
              if (do_merge) {
                float g[32];
                if (prev_branch >= 0) {
#if VKV_MERGE_RESIDUAL
                  // the earlier branch's partial: its bf16 row plus the residual row
                  load_residual32(prow + c0, mrow + c0, g);
#else
                  // exact fp32 partial of the earlier branch, stored split at its close
                  load_split32(mrow + c0, prow + c0, g);
                  store_row32(const_cast<__nv_bfloat16*>(prow) + c0, g);
#endif
#pragma unroll
                  for (int e = 0; e < 32; ++e) g[e] = c_last * f[e] + c_prev * g[e];
                } else {
#pragma unroll
                  for (int e = 0; e < 32; ++e) g[e] = c_last * f[e];
                }
                store_row32(mrow + c0, g);
              }
            }
          }
          if (row_ok) {
            p.lse[lb][(size_t)u.s * p.Lq + qrow] = has ? L_last * kLn2 : -INFINITY;
            if (do_merge)
              p.lsem[(size_t)u.s * p.Lq + qrow] =
                  (M == -INFINITY) ? -INFINITY : (Ms + lg2_approx(den)) * kLn2;
          }
        }
      }
      if (u.piece && active && ok && nsteps > 0) {
        // close the branch still open; the combine kernel that follows this grid on
        // the stream merges the unit's pieces
        tc_fence_after();
        piece_close_branch<D>(p, piece_slot(p, piece_k - 1), t, cur_branch, r, row_ok, tO, m, l);
      }
      if (ok && active && row_ok && !u.piece && (!kx || t == 0)) {
        // branches without any key tile: O = 0, LSE = -inf
        const int nb = (sparse || ragged) ? 1 : p.n_branches;
        for (int br = 0; br < nb; ++br) {
          const bool empty = (sparse || ragged) ? (nsteps == 0) : (p.branch_steps[br] == 0);
          if (!empty) continue;
          __nv_bfloat16* orow =
              p.o[br] + u.b * p.o_sb[br] + (long long)qrow * p.o_st[br] + u.h * p.o_sh[br];
          float z[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) z[e] = 0.f;
          for (int c0 = 0; c0 < D; c0 += 32) store_row32(orow + c0, z);
          p.lse[br][(size_t)u.s * p.Lq + qrow] = -INFINITY;
        }
        if (nsteps == 0 && p.om != nullptr && p.n_branches == 2 && !sparse && !ragged) {
          __nv_bfloat16* mrow = p.om + u.b * p.om_sb + (long long)qrow * p.om_st + u.h * p.om_sh;
          float z[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) z[e] = 0.f;
          for (int c0 = 0; c0 < D; c0 += 32) store_row32(mrow + c0, z);
          p.lsem[(size_t)u.s * p.Lq + qrow] = -INFINITY;
        }
      }
      if (sparse) {
        __syncwarp();
        if (lane == 0) mbar_arrive(b_lfree0 + 8 * lb);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace vkv
