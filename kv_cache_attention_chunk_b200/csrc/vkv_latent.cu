// Latent (multi-head latent) attention over a head-shared video KV cache: the
// sm_100a kernel and its C entry point.
//
// VideoMLA technical summary, "Methodology": every cached token keeps one
// head-shared row [c_t ; k^R_t] (content latent of width d_c, rotary key of
// width d_rope = 32) instead of per-head keys and values.  With the key
// up-projection absorbed into the query and the value up-projection left to
// the output projection, head h computes
//     s_t = scale * <qa_h, [c_t ; k^R_t]>,   o_h = sum_t softmax(s)_t c_t,
// i.e. attention whose keys are the cached rows and whose values are their
// first d_c columns, shared by every head.
//
// Because keys and values are the same bytes, one copy of a 128-row cache
// tile in shared memory serves both products: S = Q K^T reads it K-major
// (contraction over the row), O += P V reads its latent part MN-major
// (contraction over the tokens).  The rotary part (32 columns = 64 B per row)
// is kept in a 64-byte-swizzled block next to the latent atoms, so a tile is
// d_c/64 atoms of 16 KB plus 8 KB.
//
// One persistent CTA per SM walks query tiles (128 rows of one batch and head)
// in a fixed round robin; every tile streams all cache tiles, so all tiles
// cost the same.  Per tile the S accumulator is double-buffered in tensor
// memory, so the softmax of cache tile j overlaps S(j+1) = Q K_{j+1}^T and
// O += P(j-1) V_{j-1} on the tensor pipe:
//   TMEM columns: S_0 [0,128), S_1 [128,256), O [256, 256 + d_c).
// The softmax threads write P(j) (bf16, two per column) over the first 64
// columns of S(j mod 2); the PV MMA reads it from there (A operand in TMEM).
//
// Warp roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer (owns the
// TMEM allocation), warps 2-3 idle, warps 4-7 softmax and epilogue (one
// thread per query row; warp 4+q reads TMEM lanes [32q, 32q+32)).
//
// Ordering (every mbarrier phase is observed exactly once by its waiter, so
// parity waits cannot alias):
//   MMA    per step j: wait P(j) -> O += P(j) V_j -> commit o_done, empty[slot]
//          -> S(j+2) = Q K_{j+2}^T into the same S buffer (issue order keeps
//          P(j) read before it is overwritten) -> commit s_full.
//   softmax per step j: wait S(j) -> P(j) -> wait o_done of PV(j-1) -> rescale
//          O if the running maximum moved by more than 2^8 -> arrive P(j).
//   tile end: softmax waits the last PV, writes O / l and LSE, arrives o_free;
//          the next tile's first PV (which overwrites O) waits o_free.
#include "vkv_internal.h"
#include "vkv_ptx.cuh"
#include "vkv_tmap.h"

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <mutex>

namespace vkv {
namespace {

constexpr int kRope = 32;  // rotary key width (columns) this kernel serves

struct LatCtl {
  uint64_t full[4], empty[4];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int DC>
struct LatCfg {
  static constexpr int NAC = DC / 64;             // 16 KB atoms of the latent part
  static constexpr int ATOM = 128 * 128;          // 128 rows x 128 B
  static constexpr int ROPE = 128 * 64;           // 128 rows x 64 B (64-byte swizzle)
  static constexpr int TILE = NAC * ATOM + ROPE;  // one 128-row Q or cache tile
  static constexpr int NSLOT = (DC == 192) ? 3 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = TILE;
  static constexpr int OFF_CTL = OFF_KV + NSLOT * TILE;
  static constexpr int SMEM_BYTES = OFF_CTL + 256 + 1024;  // + base alignment slack
  static constexpr uint32_t TM_O = 256;
  // the first KQ_TS 16-column steps of the query (its first 128 latent columns)
  // also live in TMEM columns [448, 512), so that those steps of S = Q K^T run
  // in TS form (A from TMEM: ~92 cycles against ~115 in SS form)
  static constexpr int KQ_TS = 8;
  static constexpr uint32_t TM_QA = 448;
  static_assert(TM_O + DC <= TM_QA && TM_QA + 8 * KQ_TS <= 512, "tensor memory budget");
  static_assert(sizeof(LatCtl) <= 256, "control block");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(TILE % 1024 == 0, "atom alignment");
};

struct LatParams {
  CUtensorMap tm_qc;  // (d_c, H, Lq, B), box (64, 1, 128, 1), 128 B swizzle
  CUtensorMap tm_qr;  // (32, H, Lq, B), box (32, 1, 128, 1), 64 B swizzle
  CUtensorMap tm_c;   // (d_c, 1, Lkv, B), box (64, 1, 128, 1), 128 B swizzle
  CUtensorMap tm_r;   // (32, 1, Lkv, B), box (32, 1, 128, 1), 64 B swizzle
  __nv_bfloat16* o;
  long long o_sb, o_st, o_sh;
  float* lse;  // optional [B, H, Lq]
  int* err;
  int withhold_first_copy;  // test build only (vkv_debug_withhold_copy)
  int B, H, Lq, Lkv, n_qt, n_tiles;
  float scale_log2;
};

// Shared-memory matrix descriptor of a K-major operand with 64-byte swizzle
// (sm_100 layout code 4): rows of 64 B (32 bf16 along K), 8-row groups 512 B
// apart; the two 16-element K slices of a row start at +0 and +32 B.
__device__ __forceinline__ uint64_t sdesc_k_sw64(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;            // leading byte offset (unused by this layout): 16 B
  d |= (uint64_t)(512 >> 4) << 32;   // stride byte offset: 8-row group pitch
  d |= (uint64_t)1 << 46;            // descriptor version for sm_100
  d |= (uint64_t)4 << 61;            // swizzle: 64 B
  return d;
}

// Part of the exponentials can run on the FMA pipe instead of MUFU (one MUFU
// ex2 per score and one softmax warp per SM sub-partition make MUFU the
// longest part of a step): kLatExpEmu of every 16 columns.  2^x = 2^r q(f),
// r = round(x) by the 1.5 * 2^23 trick, f = x - r in [-1/2, 1/2], q a cubic
// fitted to 2^f by relative-error minimax (max relative error 7.5e-5, far below
// the 2^-9 rounding of P to bf16); 2^r enters the exponent field as an integer
// add.  Arguments below -126 give at most 2^-126 (masked scores are -inf).
#ifndef VKV_LAT_EXP_EMU
#define VKV_LAT_EXP_EMU 0
#endif
constexpr int kLatExpEmu = VKV_LAT_EXP_EMU;

__device__ __forceinline__ void lat_exp2_pair(float x0, float x1, float& e0, float& e1) {
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

// Copy a 128-row x 32-byte slice of a shared-memory matrix (matrix descriptor,
// as for an MMA operand) into 8 tensor-memory columns: lane i receives row i,
// two bf16 per 32-bit column, the layout of an A operand read from TMEM.
// Ordered with the tcgen05.mma ops issued after it by the same thread.
__device__ __forceinline__ void tmem_cp_128x256b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

constexpr float kLn2f = 0.6931471805599453f;

__device__ __forceinline__ bool lat_all(bool v) { return __all_sync(0xFFFFFFFFu, v); }
constexpr float kRescaleLog2 = 8.0f;

__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16* dst, const float* v) {
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

struct TileId {
  int b, h, qt;
};

__device__ __forceinline__ TileId tile_id(const LatParams& p, int i) {
  TileId t;
  t.qt = i % p.n_qt;
  const int bh = i / p.n_qt;
  t.b = bh / p.H;
  t.h = bh - t.b * p.H;
  return t;
}

template <int DC>
__global__ void __launch_bounds__(256, 1) latent_attn_kernel(const __grid_constant__ LatParams p) {
  using C = LatCfg<DC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  LatCtl* ctl = reinterpret_cast<LatCtl*>(smem + C::OFF_CTL);
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
  const uint32_t b_odone = smem_u32(&ctl->o_done);
  const uint32_t b_ofree = smem_u32(&ctl->o_free);
  const uint32_t b_drain = smem_u32(&ctl->drain);
  const int nsteps = (p.Lkv + 127) >> 7;

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
    }
    mbar_init(b_odone, 1);
    mbar_init(b_ofree, 4);
    mbar_init(b_drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_qc);
    tma_prefetch_desc(&p.tm_qr);
    tma_prefetch_desc(&p.tm_c);
    tma_prefetch_desc(&p.tm_r);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nsteps > 0) {
      uint32_t item = 0, qcnt = 0;
      bool ok = true;
      for (int ti = blockIdx.x; ti < p.n_tiles && ok; ti += gridDim.x) {
        const TileId t = tile_id(p, ti);
        if (qcnt > 0) ok = mbar_wait(b_qempty, (qcnt - 1) & 1, abort_flag, p.err);
        if (!ok) break;
        mbar_arrive_expect_tx(b_qfull, (uint32_t)C::TILE);
#pragma unroll
        for (int ac = 0; ac < C::NAC; ++ac)
          tma_load_4d(sQ + ac * C::ATOM, &p.tm_qc, ac * 64, t.h, t.qt * 128, t.b, b_qfull);
        tma_load_4d(sQ + C::NAC * C::ATOM, &p.tm_qr, 0, t.h, t.qt * 128, t.b, b_qfull);
        ++qcnt;
        for (int j = 0; j < nsteps; ++j) {
          const uint32_t slot = item % C::NSLOT, use = item / C::NSLOT;
          if (use > 0) ok = mbar_wait(b_empty0 + 8 * slot, (use - 1) & 1, abort_flag, p.err);
          if (!ok) break;
#ifdef VKV_TEST_AIDS
          if (item == 0 && p.withhold_first_copy) {
            ++item;  // test aid: this copy never arrives, so the wait for it runs out
            continue;
          }
#endif
          const uint32_t bar = b_full0 + 8 * slot;
          const uint32_t dst = sKV + slot * C::TILE;
          mbar_arrive_expect_tx(bar, (uint32_t)C::TILE);
#pragma unroll
          for (int ac = 0; ac < C::NAC; ++ac) tma_load_4d(dst + ac * C::ATOM, &p.tm_c, ac * 64, 0, j * 128, t.b, bar);
          tma_load_4d(dst + C::NAC * C::ATOM, &p.tm_r, 0, 0, j * 128, t.b, bar);
          ++item;
        }
      }
      if (!ok) {
        // let copies already issued land before the CTA exits
        for (uint32_t i = (item > (uint32_t)C::NSLOT ? item - C::NSLOT : 0); i < item; ++i)
          mbar_wait_drain(b_full0 + 8 * (i % C::NSLOT), (i / C::NSLOT) & 1);
        if (qcnt > 0) mbar_wait_drain(b_qfull, (qcnt - 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nsteps > 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, DC, false, true);
      uint32_t item = 0, qcnt = 0, g = 0, ucnt = 0;
      bool ok = true;
      // S(j) = Q K_j^T into S buffer (g + j) & 1
      auto issue_qk = [&](int j) -> bool {
        const uint32_t it = item + (uint32_t)j;
        if (!mbar_wait(b_full0 + 8 * (it % C::NSLOT), (it / C::NSLOT) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
        const uint32_t sb = (g + (uint32_t)j) & 1u;
        const uint32_t d_tm = tmem + sb * 128u;
        const uint32_t kb = sKV + (it % C::NSLOT) * C::TILE;
#pragma unroll
        for (int kk = 0; kk < DC / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM + (kk & 3) * 32;
          if (kk < C::KQ_TS)
            mma_bf16_ts(d_tm, tmem + C::TM_QA + 8 * kk, sdesc_k_sw128(kb + off), IDESC_QK, kk > 0);
          else
            mma_bf16_ss(d_tm, sdesc_k_sw128(sQ + off), sdesc_k_sw128(kb + off), IDESC_QK, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < kRope / 16; ++kk) {
          const uint32_t off = C::NAC * C::ATOM + kk * 32;
          mma_bf16_ss(d_tm, sdesc_k_sw64(sQ + off), sdesc_k_sw64(kb + off), IDESC_QK, 1u);
        }
        mma_commit(b_sfull0 + 8 * sb);
        if (j == nsteps - 1) mma_commit(b_qempty);  // Q is read by the tile's QK products only
        return true;
      };
      for (int ti = blockIdx.x; ti < p.n_tiles && ok; ti += gridDim.x, ++ucnt) {
        ok = mbar_wait(b_qfull, qcnt & 1, abort_flag, p.err);
        ++qcnt;
        if (!ok) break;
        tc_fence_after();
        // the tile's query slices for the TS steps -> TMEM (in order with the MMAs below;
        // the previous tile's QK products, issued earlier, have read the old ones)
#pragma unroll
        for (int kk = 0; kk < C::KQ_TS; ++kk)
          tmem_cp_128x256b(tmem + C::TM_QA + 8 * kk, sdesc_k_sw128(sQ + (kk >> 2) * C::ATOM + (kk & 3) * 32));
        ok = issue_qk(0);
        if (ok && nsteps > 1) ok = issue_qk(1);
        for (int j = 0; j < nsteps && ok; ++j) {
          const uint32_t G = g + (uint32_t)j, sb = G & 1u;
          ok = mbar_wait(b_pfull0 + 8 * sb, (G >> 1) & 1, abort_flag, p.err);
          if (ok && j == 0 && ucnt > 0) ok = mbar_wait(b_ofree, (ucnt - 1) & 1, abort_flag, p.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t slot = (item + (uint32_t)j) % C::NSLOT;
          const uint32_t vb = sKV + slot * C::TILE;
          const uint32_t pa = tmem + sb * 128u;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + C::TM_O, pa + 8 * kk, sdesc_mn_sw128(vb + kk * 2048, C::ATOM), IDESC_PV,
                        (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(b_odone);
          mma_commit(b_empty0 + 8 * slot);
          if (j + 2 < nsteps) ok = issue_qk(j + 2);
        }
        item += (uint32_t)nsteps;
        g += (uint32_t)nsteps;
      }
      // every MMA issued so far completes before TMEM is released
      mma_commit(b_drain);
      mbar_wait_drain(b_drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + (int)lane;  // row inside the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_base + C::TM_O;
    const float sl2 = p.scale_log2;
    uint32_t g = 0, ucnt = 0;
    bool ok = true;
    for (int ti = blockIdx.x; ti < p.n_tiles && ok; ti += gridDim.x, ++ucnt) {
      const TileId t = tile_id(p, ti);
      const int qrow = t.qt * 128 + r;
      const bool row_ok = qrow < p.Lq;
      __nv_bfloat16* orow = p.o + t.b * p.o_sb + (long long)qrow * p.o_st + t.h * p.o_sh;
      float* lrow = p.lse ? p.lse + ((size_t)t.b * p.H + t.h) * p.Lq + qrow : nullptr;
      if (nsteps == 0) {
        // empty cache: O = 0, LSE = -inf
        if (row_ok) {
          float z[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) z[e] = 0.f;
#pragma unroll
          for (int c0 = 0; c0 < DC; c0 += 32) store_row32_bf16(orow + c0, z);
          if (lrow) *lrow = -INFINITY;
        }
        continue;
      }
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nsteps; ++j) {
        const uint32_t G = g + (uint32_t)j, sb = G & 1u;
        const uint32_t tS = tmem + lane_base + sb * 128u;
        ok = lat_all(mbar_wait(b_sfull0 + 8 * sb, (G >> 1) & 1, abort_flag, p.err));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(tS + 0, sr + 0);
        tmem_ld32(tS + 32, sr + 32);
        tmem_ld32(tS + 64, sr + 64);
        tmem_ld32(tS + 96, sr + 96);
        tmem_ld_wait();
        reg_fence<128>(sr);
        // cache rows past Lkv (zero-filled by the copy) are masked
        const int lim = p.Lkv - j * 128;
        if (lim < 128) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          mx8[i] = max3f(__uint_as_float(sr[i]), __uint_as_float(sr[8 + i]), __uint_as_float(sr[16 + i]));
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
        float alpha = 1.f;
        bool rescale = false;
        if (m == -INFINITY) {
          m = mt;
        } else if (mt > m + kRescaleLog2) {
          alpha = ex2_approx(m - mt);
          m = mt;
          rescale = true;
        }
        const float mu = (m == -INFINITY) ? 0.f : m;
        // p = 2^(s * scale * log2 e - m); P (bf16 pairs) -> the first 64 columns of S
        const uint64_t sl2x2 = pack2f(sl2, sl2), nmu2 = pack2f(-mu, -mu);
        uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[32];
#pragma unroll
          for (int gg = 0; gg < 64; gg += 16) {
            const int c0 = hh * 64 + gg;
            float a[16], e[16];
#pragma unroll
            for (int i = 0; i < 16; i += 2)
              unpack2f(fma2f(pack2f(__uint_as_float(sr[c0 + i]), __uint_as_float(sr[c0 + i + 1])), sl2x2, nmu2),
                       a[i], a[i + 1]);
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              if (i >= 16 - kLatExpEmu) {
                lat_exp2_pair(a[i], a[i + 1], e[i], e[i + 1]);
              } else {
                e[i] = ex2_approx(a[i]);
                e[i + 1] = ex2_approx(a[i + 1]);
              }
            }
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              acc2[(i >> 1) & 3] = add2f(acc2[(i >> 1) & 3], pack2f(e[i], e[i + 1]));
              pk[(gg + i) >> 1] = pack_bf16x2(e[i], e[i + 1]);
            }
          }
          tmem_st32(tS + (uint32_t)(hh * 32), pk);
        }
        float sum_lo, sum_hi;
        unpack2f(add2f(add2f(acc2[0], acc2[1]), add2f(acc2[2], acc2[3])), sum_lo, sum_hi);
        l = l * alpha + (sum_lo + sum_hi);
        if (j > 0) {
          // O holds exactly PV(0..j-1) once PV(j-1) is done; PV(j) waits for P(j)
          ok = lat_all(mbar_wait(b_odone, (G - 1) & 1, abort_flag, p.err));
          if (!ok) break;
          tc_fence_after();
          if (__any_sync(0xFFFFFFFFu, rescale)) {
#pragma unroll
            for (int c0 = 0; c0 < DC; c0 += 32) {
              uint32_t v[32];
              tmem_ld32(tO + c0, v);
              tmem_ld_wait();
              reg_fence<32>(v);
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
              tmem_st32(tO + c0, v);
            }
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_pfull0 + 8 * sb);
      }
      if (ok) ok = lat_all(mbar_wait(b_odone, (g + (uint32_t)nsteps - 1) & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const bool has = l > 0.f;
      const float inv = has ? 1.f / l : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < DC; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tO + c0, v);
        tmem_ld_wait();
        reg_fence<32>(v);
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]) * inv;
        if (row_ok) store_row32_bf16(orow + c0, f);
      }
      if (row_ok && lrow) *lrow = has ? (m + lg2_approx(l)) * kLn2f : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_ofree);
      g += (uint32_t)nsteps;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

bool lat_aligned(const vkv_tensor& t) {
  return t.ptr != nullptr && tensor_aligned(t);
}

// (w, H, L, B) map of the columns [col0, col0 + w) of a [B, L, H, *] tensor.
bool encode_lat(CUtensorMap* tm, const void* ptr, long long sb, long long st, long long sh, int B, int L,
                int H, int w, int box_w, int swz) {
  const uint64_t dims[4] = {(uint64_t)w, (uint64_t)H, (uint64_t)L, (uint64_t)B};
  const uint64_t bsh = (H == 1) ? (uint64_t)st * 2 : (uint64_t)sh * 2;
  const uint64_t bst = (uint64_t)st * 2;
  const uint64_t bsb = (B == 1) ? bst * (uint64_t)L : (uint64_t)sb * 2;
  const uint64_t strides[3] = {bsh, bst, bsb};
  const uint32_t box[4] = {(uint32_t)box_w, 1, 128, 1};
  return encode_tmap_bf16_4d_swizzle(tm, ptr, dims, strides, box, swz);
}

template <int DC>
bool lat_prepare(int dev) {
  static std::mutex mu;
  static unsigned long long done = 0;
  std::lock_guard<std::mutex> lk(mu);
  if (done & (1ull << dev)) return true;
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(latent_attn_kernel<DC>),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, LatCfg<DC>::SMEM_BYTES) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  done |= 1ull << dev;
  return true;
}

}  // namespace
}  // namespace vkv

extern "C" vkv_status vkv_latent_attn(const vkv_latent_args* a, vkv_stream_t stream) {
  using namespace vkv;
  if (!a) return VKV_ERR_NULL;
  if (a->B <= 0 || a->H <= 0 || a->Lq <= 0 || a->Lkv < 0) return VKV_ERR_SHAPE;
  if (a->d_rope != kRope || (a->d_c != 128 && a->d_c != 192)) return VKV_ERR_UNSUPPORTED;
  if ((long long)a->B * a->H * ((a->Lq + 127) / 128) > (1ll << 30)) return VKV_ERR_SHAPE;
  const bool has_kv = a->Lkv > 0;
  if (!a->q.ptr || !a->o.ptr || (has_kv && !a->kv.ptr)) return VKV_ERR_NULL;
  if (!(a->scale > 0.f) || !std::isfinite(a->scale)) return VKV_ERR_SHAPE;
  const bool sep_rope = a->kr.ptr != nullptr;
  if (!lat_aligned(a->q) || !lat_aligned(a->o) || (has_kv && !lat_aligned(a->kv)) ||
      (has_kv && sep_rope && !lat_aligned(a->kr)))
    return VKV_ERR_ALIGN;
  const long long lim = 1ll << 39;
  auto strides_ok = [&](const vkv_tensor& t, bool heads) {
    return std::llabs(t.sb) < lim && std::llabs(t.st) < lim && std::llabs(t.sh) < lim && t.st > 0 &&
           (a->B == 1 || t.sb > 0) && (!heads || a->H == 1 || t.sh > 0);
  };
  if (!strides_ok(a->q, true) || !strides_ok(a->o, true)) return VKV_ERR_SHAPE;
  if (has_kv && (!strides_ok(a->kv, false) || (sep_rope && !strides_ok(a->kr, false)))) return VKV_ERR_SHAPE;

  int dev = 0;
  const int n_sm = device_sm_count(&dev);
  if (n_sm <= 0) return VKV_ERR_CUDA;

  LatParams P{};
  const int dc = a->d_c;
  const uint8_t* q8 = static_cast<const uint8_t*>(a->q.ptr);
  if (!encode_lat(&P.tm_qc, q8, a->q.sb, a->q.st, a->q.sh, a->B, a->Lq, a->H, dc, 64, 128) ||
      !encode_lat(&P.tm_qr, q8 + 2 * (size_t)dc, a->q.sb, a->q.st, a->q.sh, a->B, a->Lq, a->H, kRope, kRope, 64))
    return VKV_ERR_CUDA;
  if (has_kv) {  // the maps of an empty cache are never read
    const uint8_t* kv8 = static_cast<const uint8_t*>(a->kv.ptr);
    const vkv_tensor& rt = sep_rope ? a->kr : a->kv;
    const uint8_t* r8 = sep_rope ? static_cast<const uint8_t*>(a->kr.ptr) : kv8 + 2 * (size_t)dc;
    if (!encode_lat(&P.tm_c, kv8, a->kv.sb, a->kv.st, a->kv.st, a->B, a->Lkv, 1, dc, 64, 128) ||
        !encode_lat(&P.tm_r, r8, rt.sb, rt.st, rt.st, a->B, a->Lkv, 1, kRope, kRope, 64))
      return VKV_ERR_CUDA;
  }
  P.o = reinterpret_cast<__nv_bfloat16*>(a->o.ptr);
  P.o_sb = a->o.sb;
  P.o_st = a->o.st;
  P.o_sh = a->o.sh;
  P.lse = a->lse;
  P.err = a->err_word;
#ifdef VKV_TEST_AIDS
  P.withhold_first_copy = take_withhold_request() ? 1 : 0;
#endif
  P.B = a->B;
  P.H = a->H;
  P.Lq = a->Lq;
  P.Lkv = a->Lkv;
  P.n_qt = (a->Lq + 127) / 128;
  P.n_tiles = a->B * a->H * P.n_qt;
  P.scale_log2 = a->scale * 1.4426950408889634f;
  const int grid = std::min(P.n_tiles, n_sm);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dc == 192) {
    if (!lat_prepare<192>(dev)) return VKV_ERR_CUDA;
    latent_attn_kernel<192><<<grid, 256, LatCfg<192>::SMEM_BYTES, st>>>(P);
  } else {
    if (!lat_prepare<128>(dev)) return VKV_ERR_CUDA;
    latent_attn_kernel<128><<<grid, 256, LatCfg<128>::SMEM_BYTES, st>>>(P);
  }
  if (cudaGetLastError() != cudaSuccess) return VKV_ERR_CUDA;
  return VKV_OK;
}
