// Internal declarations shared by the host launchers and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "vkv.h"

namespace vkv {

constexpr int kMaxUnits = 6144;        // work units per launch (kernel parameter space)
constexpr int kMaxCtas = 160;          // >= SMs of a B200 (148)
constexpr int kMaxListEntries = 288;   // block list of one BLOCK_SPARSE unit
constexpr int kCtlBytes = 2048;        // control block in shared memory
constexpr int kMaxFlatSegs = VKV_MAX_BRANCHES * VKV_MAX_SEGMENTS;
constexpr int kMaxPieces = 384;        // key-axis pieces per launch (kernel parameter space)
constexpr int kMaxPiecesPerUnit = 8;   // pieces one split unit may be cut into
constexpr int kMaxSplitUnits = kMaxPieces / 2;  // split units per launch (each has >= 2 pieces)

// Kernel parameters of the attention kernel, passed as __grid_constant__.
// Unit code: bits [0,12) first query tile, bit 12 piece (the unit covers only the
// key steps of its piece entry), bit 13 two tiles, bits [14,32) sequence b*H+h.
//
// Piece entry (uint2): x = first step | end step << 16 (key-tile steps of the
// unit's stream); y = first workspace slot of the unit | piece index << 16 |
// piece count << 24.  The piece entries of CTA c are pieces[cta_piece0[c] ..],
// in the order its unit list meets them.
struct AttnParams {
  CUtensorMap tm_q;  // dims (d, H, Lq, B); box (64, 1, 128 or 64 (BLOCK_SPARSE), 1); 128 B swizzle
  CUtensorMap tm_k;  // dims (d, H, Lkv, B) or (d, 1, rows, 1); box (64, 1, 64, 1)
  CUtensorMap tm_v;
  int mode, B, H, Lq, Lkv, d;
  float scale_log2;  // softmax scale * log2(e)
  int n_branches;
  int branch_steps[VKV_MAX_BRANCHES];
  int total_steps;
  int n_flat;  // SEGMENTS: non-empty segments in branch order
  int flat_start[kMaxFlatSegs];
  int flat_len[kMaxFlatSegs];
  int flat_branch[kMaxFlatSegs];
  int flat_first[kMaxFlatSegs];
  int flat_step0[kMaxFlatSegs];  // first key-tile step of each flat segment
  // BLOCK_SPARSE
  int n_persist, topk, window_blk0, n_win_blk, n_qblk, n_blocks_total;
  const int* persist_idx;
  const int* sel_idx;
  const int* qblk_order;  // optional [B*H][n_qblk] query-block permutation
  // BLOCK_SPARSE with the selection in the kernel: the queries (elements, strides
  // in elements), the window block means [B*H][n_win_blk][d] and where the
  // selection goes (optional, [B*H][n_qblk][topk])
  const __nv_bfloat16* qp;
  long long q_sb, q_st, q_sh;
  const float* kbar;
  int* sel_out;
  // RAGGED
  const int* cu_seqlens;
  // outputs
  __nv_bfloat16* o[VKV_MAX_BRANCHES];
  long long o_sb[VKV_MAX_BRANCHES], o_st[VKV_MAX_BRANCHES], o_sh[VKV_MAX_BRANCHES];
  float* lse[VKV_MAX_BRANCHES];
  __nv_bfloat16* om;
  long long om_sb, om_st, om_sh;
  float* lsem;
  int* err;
  int withhold_first_copy;  // test build only: the producer skips its first K/V copy (vkv_debug_withhold_copy)
  // key-axis pieces: per workspace slot, the partial outputs (O / l, fp32)
  // [slot][tile 2][branch n_branches][row 128][d] and their LSEs (natural log)
  // [slot][tile][branch][row]
  int sp_est[2];  // BLOCK_SPARSE: key steps the schedule assumed for a 1- / 2-tile unit
  // BLOCK_SPARSE with the selection in the kernel: a one-tile unit splits its key tiles
  // between the two softmax warpgroups (even steps S_0/O_0, odd steps S_1/O_1) and
  // merges the two by LSE
  int kx;
  float* ws_o;
  float* ws_l;
  // schedule: CTA c runs units[cta_begin[c] .. cta_begin[c+1])
  int n_ctas;
  int cta_begin[kMaxCtas + 1];
  int cta_piece0[kMaxCtas + 1];
  uint2 pieces[kMaxPieces];
  uint32_t units[kMaxUnits];
};

// Parameters of the piece combine kernel: the split units of one attention launch
// (code = the unit code without the piece bit; slots = first workspace slot |
// piece count << 16) and where their outputs go.
struct CombineParams {
  int mode, H, Lq, n_qblk, nbr;
  const int* qblk_order;
  const float* ws_o;
  const float* ws_l;
  __nv_bfloat16* o[VKV_MAX_BRANCHES];
  long long o_sb[VKV_MAX_BRANCHES], o_st[VKV_MAX_BRANCHES], o_sh[VKV_MAX_BRANCHES];
  float* lse[VKV_MAX_BRANCHES];
  __nv_bfloat16* om;
  long long om_sb, om_st, om_sh;
  float* lsem;
  int n_units;
  uint32_t code[kMaxSplitUnits];
  uint32_t slots[kMaxSplitUnits];
};

// Host helpers (vkv_common.cu).
int device_sm_count(int* dev_out);                // -1 when no usable sm_100 device
bool encode_tmap_bf16_4d(CUtensorMap* tm, const void* ptr, const uint64_t dims[4],
                         const uint64_t strides_bytes[3], const uint32_t box[4]);
bool tensor_aligned(const vkv_tensor& t);
#ifdef VKV_TEST_AIDS
// Test aid (vkv_common.cu, test build only): true when the calling launch should
// withhold its first cache-tile copy (consumes one of the calls armed by
// vkv_debug_withhold_copy).
bool take_withhold_request();
#endif

}  // namespace vkv
