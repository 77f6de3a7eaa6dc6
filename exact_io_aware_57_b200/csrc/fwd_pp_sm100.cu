// Forward attention on sm_100a tensor cores, two query tiles per CTA.
//
// One CTA owns 256 query rows of one (batch or sequence, head), as two tiles
// of 128 rows, and streams 128-key tiles of K and V past both ("Attention IO
// tiling" lesson card, The mechanism: tiles staged on chip, each score block
// folded into the per-row softmax state and then dropped).  Each tile has its
// own softmax warpgroup, so while one warpgroup exponentiates the scores of
// its tile the tensor pipe multiplies for the other ("Understanding
// FlashAttention Pt 1", contents 5.5: overlap data movement, matrix products
// and the softmax).
//
//   warps 0..3  softmax of tile 0: thread r owns query row r (TMEM lane r)
//   warps 4..7  softmax of tile 1
//   warp 8      TMEM owner + single-thread tcgen05.mma issuer
//   warp 9      TMA producer: Q_0, Q_1 once, then K_j, V_j into smem rings
//
// TMEM (512 columns x 128 lanes x 32 bit):
//   [  0,128) S_0 = Q_0 K_j^T (fp32); P_0 (bf16 pairs) over its first 64 columns
//   [128,256) S_1, P_1 likewise
//   [256,256+DV) O_0,  [256+DV,256+2DV) O_1   (fp32 accumulators)
//
// MMA issue order per key tile j (tile t only where j is in its key range):
//   O_0 += P_0 V_j;  S_0 = Q_0 K_{j+1}^T;  O_1 += P_1 V_j;  S_1 = Q_1 K_{j+1}^T
// tcgen05.mma executes in issue order, so S_t of step j+1 overwrites P_t only
// after P_t V_j has read it, and the commit that announces S_t of step j+1
// also covers P_t V_j: when a softmax thread sees its scores it may rescale
// its O rows at once, without a separate wait.
//
// Per key tile the softmax thread of row i forms x = s * scale * log2(e)
// (+ bias * log2(e)), moves its reference max m only when the tile max
// exceeds m by more than 2^8 (the final O / l and LSE do not depend on the
// reference), p = 2^(x - m), l = 2^(m_old - m) l + sum p ("Softmax does not
// need the matrix", "Carry the Normalizer", in base 2), writes P over the
// scores it has read, rescales its O row by 2^(m_old - m) when m moved, and
// hands the tile to the MMA warp.  After the last tile it writes O / l and
// LSE = (m + log2 l) ln 2.
// Causal and local attention load only the key tiles meeting a tile's visible
// band and mask only the tiles on its edges ("Understanding FlashAttention Pt
// 1", contents 3.5 and 4.2); the two tiles' key ranges are contiguous and
// nested at their ends, and each tile walks only its own.
// Split-KV: with num_splits > 1 the grid's z index also runs over key ranges;
// each CTA then writes O_t (normalised, fp32) and LSE_t for the merge.
// With equal units, a last wave that would fill at most half the SMs runs its
// 256-row units as single 128-row tiles, one CTA each (FwdParams::half_from).
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace attn {

namespace {

constexpr int BM = 128;  // query rows per tile (two tiles per CTA)
constexpr int BN = 128;  // keys per KV tile
#ifndef ATTN_FWD_REG_SPLIT
#define ATTN_FWD_REG_SPLIT 0
#endif
// Register split: 12 warps launched at 168 registers a thread (384 x 168 =
// 64,512 of the 65,536); warps 8..11 (MMA, TMA, two idle) give theirs down to
// 88 and the two softmax warpgroups take 208: 4 x 32 x 88 + 8 x 32 x 208 =
// 64,512, the launch's pool, and per SM sub-partition (three warps) 2 x 32 x
// 208 + 32 x 88 = 16,128 of its 16,384.  Without it: 10 warps, 168 registers.
constexpr bool kRegSplit = ATTN_FWD_REG_SPLIT != 0;
constexpr int kThreads = kRegSplit ? 384 : 320;
constexpr int kLaunchRegs = 168, kLowRegs = 88, kHighRegs = 208;
static_assert(!kRegSplit || (4 * 32 * kLowRegs + 8 * 32 * kHighRegs == kThreads * kLaunchRegs &&
                             2 * 32 * kHighRegs + 32 * kLowRegs <= 16384),
              "register split must match the launch's pool");
constexpr int kWarpMma = 8, kWarpLoad = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.f;  // log2 units: P stays <= 256
#ifndef ATTN_EX2_EMU_EVERY
#define ATTN_EX2_EMU_EVERY 0
#endif
// One bf16 pair of P in kEmuEvery is exponentiated on the FMA pipe (0: none).
constexpr int kEmuEvery = ATTN_EX2_EMU_EVERY;

// K/V ring depth: as many stages as fit beside the two Q tiles in ~220 KB.
// QK8: Q and K held as e4m3 (one byte per element) for the FP8 forward.
template <int D, int DV, bool QK8>
constexpr int kStages = QK8 ? 3 : (D == 128 && DV == 128) ? 2 : (D == 64 && DV == 64) ? 4 : 3;

template <int D, int DV, bool QK8 = false>
struct PPSmem {
  static constexpr int NST = kStages<D, DV, QK8>;
  static constexpr int kQBytes = BM * D * (QK8 ? 1 : 2);
  static constexpr int kKBytes = BN * D * (QK8 ? 1 : 2);
  static constexpr int kVBytes = BN * DV * 2;
  alignas(1024) uint8_t q[2][kQBytes];
  alignas(1024) uint8_t k[NST][kKBytes];
  alignas(1024) uint8_t v[NST][kVBytes];
  uint64_t q_full;
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int N>
ATTN_DEVINL void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// Key-tile range of one query tile: tiles jb .. jb + n - 1 hold every key
// visible from its rows [mt, min(mt + BM, len_q)), clipped to [k_lo, k_hi).
struct TileRange {
  int jb, n;
};

ATTN_DEVINL TileRange tile_range(int mt, int len_q, int diag, int win_l, int win_r, int k_lo, int k_hi) {
  TileRange r{0, 0};
  if (mt >= len_q) return r;
  const int rows_end = min(mt + BM, len_q);
  // |mt|, |diag| < 2^28 and win_* <= 2^30: no int overflow
  const int kv_end = min(k_hi, rows_end + diag + win_r);
  const int kv_begin = max(k_lo, mt + diag - win_l);
  if (kv_end <= kv_begin) return r;
  r.jb = kv_begin / BN;
  r.n = (kv_end + BN - 1) / BN - r.jb;
  return r;
}

ATTN_DEVINL bool in_range(const TileRange& r, int j) { return r.n > 0 && j >= r.jb && j < r.jb + r.n; }

// 10 warps: three of them share one SM sub-partition's 16K registers, so a
// thread gets at most 168.
template <int D, int DV, int BIAS, bool FAST, bool PARTIAL, bool QK8 = false>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Smem = PPSmem<D, DV, QK8>;
  constexpr int NST = Smem::NST;
  constexpr int KB = D * (QK8 ? 1 : 2) / 128;  // 128-byte blocks per Q/K row
  constexpr int kBoxCols = QK8 ? 128 : 64;     // elements in one 128-byte block
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work: heavy (late) row blocks first under causal masking
  // grid (row block, head, batch [x split]); the row blocks of groups of eight
  // (batch, head) pairs are interleaved (grouped_unit).  When the batch
  // elements share a dense bias (grid (batch, row block, head)), a group is
  // every batch element of two heads, so the ones reading the same bias rows
  // run side by side
  const bool bi = !PARTIAL && p.batch_inner;
  const int nblk = bi ? (int)gridDim.y : PARTIAL ? (int)gridDim.x : p.grid_nblk;
  int blk_raw, h, z, half = -1;  // half >= 0: this CTA takes only that 128-row tile of its unit
  if (PARTIAL) {
    blk_raw = blockIdx.x, h = blockIdx.y, z = blockIdx.z / p.num_splits;
  } else if (bi) {
    const int nb = (int)gridDim.x;
    int u;
    grouped_unit(nblk, nb * p.Hq, 2 * nb, blk_raw, u);
    h = u / nb, z = u % nb;
  } else {
    int unit = linear_block(), u;
    if (unit >= p.half_from) {
      half = (unit - p.half_from) & 1;
      unit = p.half_from + ((unit - p.half_from) >> 1);
    }
    grouped_unit_at(unit, nblk, p.grid_nu, 8, blk_raw, u);
    h = u % p.Hq, z = u / p.Hq;
  }
  const int blk = p.causal ? nblk - 1 - blk_raw : blk_raw;
  const int split = PARTIAL ? (int)blockIdx.z % p.num_splits : 0;
  int q_off = 0, len_q = p.Nq, k_off = 0, len_k = p.Nk, bidx = z;
  if (p.cu_q) {
    // invalid offsets: reported in the status word, nothing read or written
    if (!packed_seq(p.cu_q, z, p.Nq, p.max_nq, p.status, q_off, len_q) ||
        !packed_seq(p.cu_k, z, p.Nk, p.max_nk, p.status, k_off, len_k))
      return;
    bidx = 0;
  }
  const int m0 = blk * 2 * BM + (half > 0 ? BM : 0);
  if (m0 >= len_q) return;  // uniform: before any barrier or TMEM use
  const int hk = h / (p.Hq / p.Hkv);
  const int diag = len_k - len_q;  // row i is aligned with key i + diag
  const int k_lo = PARTIAL ? split * p.split_len : 0;
  const int k_hi = PARTIAL ? min(len_k, (split + 1) * p.split_len) : len_k;
  TileRange rg[2];
  rg[0] = tile_range(m0, len_q, diag, p.win_l, p.win_r, k_lo, k_hi);
  rg[1] = tile_range(m0 + BM, len_q, diag, p.win_l, p.win_r, k_lo, k_hi);
  if (half >= 0) rg[1] = TileRange{0, 0};  // a single tile
  // union of the two ranges (contiguous: each tile's band overlaps the next)
  const int J0 = rg[0].n > 0 ? rg[0].jb : rg[1].jb;
  const int J1 = rg[1].n > 0 ? rg[1].jb + rg[1].n : rg[0].jb + rg[0].n;
  const int n_union = (rg[0].n > 0 || rg[1].n > 0) ? J1 - J0 : 0;

  // ---- setup
  if (threadIdx.x == 0) {
    s.abort_flag = 0;
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.v_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.p_full[t], 4);
      mbar_init(&s.o_done[t], 1);
    }
    mbar_init(&s.drain, 1);
    fence_mbar_init();
  }
  if (warp == kWarpMma) tmem_alloc(&s.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const Abort ab{&s.abort_flag, p.status, p.wait_limit};

  if (warp == kWarpLoad) {
    if constexpr (kRegSplit) setmaxnreg_dec<kLowRegs>();
    // ===================================================== TMA producer
    if (lane == 0 && n_union > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int nq = (rg[0].n > 0) + (rg[1].n > 0);
      mbar_expect_tx(&s.q_full, nq * Smem::kQBytes);
      for (int t = 0; t < 2; ++t) {
        if (rg[t].n == 0) continue;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
          tma_load_4d(s.q[t] + kb * BM * 128, &tm_q, &s.q_full, kb * kBoxCols, h, q_off + m0 + t * BM, bidx);
      }
      int issued_k = 0, issued_v = 0;
      for (int i = 0; i < n_union; ++i) {
        const int st = i % NST;
        const uint32_t ph = (i / NST) & 1;
        const int row = k_off + (J0 + i) * BN;
        if (!mbar_wait(&s.k_empty[st], ph ^ 1, ab)) break;
        mbar_expect_tx(&s.k_full[st], Smem::kKBytes);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
          tma_load_4d(s.k[st] + kb * BN * 128, &tm_k, &s.k_full[st], kb * kBoxCols, hk, row, bidx);
        ++issued_k;
        if (!mbar_wait(&s.v_empty[st], ph ^ 1, ab)) break;
        mbar_expect_tx(&s.v_full[st], Smem::kVBytes);
#pragma unroll
        for (int kb = 0; kb < DV / 64; ++kb)
          tma_load_4d(s.v[st] + kb * BN * 128, &tm_v, &s.v_full[st], kb * 64, hk, row, bidx);
        ++issued_v;
      }
      if (s.abort_flag) {
        // leave no copy in flight into shared memory that is about to be released
        mbar_wait_drain(&s.q_full, 0, p.wait_limit);
        for (int i = max(0, issued_k - NST); i < issued_k; ++i)
          mbar_wait_drain(&s.k_full[i % NST], (i / NST) & 1, p.wait_limit);
        for (int i = max(0, issued_v - NST); i < issued_v; ++i)
          mbar_wait_drain(&s.v_full[i % NST], (i / NST) & 1, p.wait_limit);
      }
    }
  } else if (warp == kWarpMma) {
    if constexpr (kRegSplit) setmaxnreg_dec<kLowRegs>();
    // ===================================================== MMA issuer
    if (lane == 0 && n_union > 0) {
      constexpr uint32_t idesc_s = idesc_bf16(BM, BN, 0, 0);   // Q_t: K-major, K_j: K-major
      constexpr uint32_t idesc_pv = idesc_bf16(BM, DV, 0, 1);  // P_t: TMEM, V_j: MN-major
      // S_t = Q_t K_j^T into columns [128 t, 128 t + 128).  K_j is released
      // once its last user has been issued (tile 0's S always precedes tile 1's).
      auto issue_s = [&](int t, int j) -> bool {
        const int i = j - J0, st = i % NST;
        if (!mbar_wait(&s.k_full[st], (i / NST) & 1, ab)) return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(s.q[t]), k_addr = smem_u32(s.k[st]);
        // one instruction per 32 bytes of the rows: K = 16 (bf16) or 32 (e4m3) elements
#pragma unroll
        for (int kk = 0; kk < KB * 4; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          if constexpr (QK8)
            mma_ss_f8(tmem + t * 128, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024),
                      idesc_e4m3(BM, BN), kk > 0);
          else
            mma_ss(tmem + t * 128, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024), idesc_s,
                   kk > 0);
        }
        mma_commit(&s.s_full[t]);
        if (t == 1 || !in_range(rg[1], j)) mma_commit(&s.k_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&s.q_full, 0, ab);
      if (rg[0].n > 0 && rg[0].jb == J0) ok = issue_s(0, J0);
      if (ok && rg[1].n > 0 && rg[1].jb == J0) ok = issue_s(1, J0);
      for (int j = J0; ok && j < J1; ++j) {
        const int i = j - J0, st = i % NST;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok) break;
          if (in_range(rg[t], j)) {
            const int step = j - rg[t].jb;
            if (!(ok = mbar_wait(&s.p_full[t], step & 1, ab))) break;
            if (!(ok = mbar_wait(&s.v_full[st], (i / NST) & 1, ab))) break;
            tc_fence_after();
            const uint32_t v_addr = smem_u32(s.v[st]);
            // O_t += P_t V_j (P_t from TMEM over S_t's first 64 columns)
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              mma_ts(tmem + 256 + t * DV, tmem + t * 128 + kk * 8, sdesc_sw128(v_addr + kk * 2048, BN * 128, 1024),
                     idesc_pv, (step > 0 || kk > 0));
            if (t == 1 || !in_range(rg[1], j)) mma_commit(&s.v_empty[st]);
            if (step == rg[t].n - 1) mma_commit(&s.o_done[t]);
            if (in_range(rg[t], j + 1)) ok = issue_s(t, j + 1);
          } else if (rg[t].n > 0 && rg[t].jb == j + 1) {
            ok = issue_s(t, j + 1);  // tile t's range starts at the next key tile
          }
        }
      }
      // TMEM must be quiescent before it is released
      mma_commit(&s.drain);
      mbar_wait_drain(&s.drain, 0, p.wait_limit);
    }
  } else if (warp < 8) {
    if constexpr (kRegSplit) setmaxnreg_inc<kHighRegs>();
    // ===================================================== softmax warpgroups
    const int t = warp >> 2;       // query tile of this warpgroup
    const int quarter = warp & 3;  // TMEM lanes [32 quarter, 32 quarter + 32)
    const int r = quarter * 32 + lane;
    const int mt = m0 + t * BM;
    const int i = mt + r;  // row inside its sequence
    // a CTA that takes a single tile (half >= 0) owns no rows of tile 1: those
    // belong to the CTA of the other half (or the next row block)
    const bool row_ok = i < len_q && !(half >= 0 && t == 1);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t col_s = tmem + lane_off + t * 128, col_o = tmem + lane_off + 256 + t * DV;
    const TileRange my = t ? rg[1] : rg[0];
    const float* brow = nullptr;  // rows past the end read the last row (their output is dropped)
    if constexpr (BIAS == kBiasDense)
      brow = p.bias + bidx * p.bias_bstride + ((long long)h * p.Nq + min(i, len_q - 1)) * p.Nk;
    float neg_slope2 = 0.f;  // ALiBi: B = -slope |key - (i + diag)|, in log2 units
    if constexpr (BIAS == kBiasAlibi) neg_slope2 = -__ldg(p.alibi + h) * kLog2e;
    // log2(e) * scale, times the e4m3 scales of this (batch, head) of Q and K in the FP8 forward
    float sc2 = p.scale_log2;
    if constexpr (QK8) sc2 *= __ldg(p.q_scale + bidx * p.Hq + h) * __ldg(p.k_scale + bidx * p.Hkv + hk);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int step = 0; step < my.n; ++step) {
      ok = __all_sync(0xffffffffu, mbar_wait(&s.s_full[t], step & 1, ab));
      if (!ok) break;
      tc_fence_after();
      const int kbase = (my.jb + step) * BN;
      // tile on an edge of the visible band, or ragged: keys outside [lo, hi) are hidden
      const bool edge =
          (kbase + BN > len_k) || (kbase + BN - 1 > mt + diag + p.win_r) || (kbase < mt + BM - 1 + diag - p.win_l);
      const int hi = min(len_k, i + diag + p.win_r + 1) - kbase;
      const int lo = i + diag - p.win_l - kbase;
      float alpha, m_next, rs0 = 0.f, rs1 = 0.f;
      // every score of the row in registers (one TMEM pass): x = s * scale * log2(e)
      // (+ bias * log2(e)) in the general case; the FAST case defers the scale
      uint32_t sr[BN];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(col_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      reg_fence(sr);
      if constexpr (BIAS == kBiasDense) {
        // the next tile's bias row into L2 while this tile is worked on
        // (four 128-byte lines, clamped inside the row)
        if (step + 1 < my.n) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(brow + min(kbase + BN + 32 * u, len_k - 1)));
        }
      }
      if constexpr (BIAS == kBiasDense) {
        // whole tiles of 16-byte aligned rows as float4 (a lane reads its own
        // row, so a warp load touches 32 rows: 16 bytes each instead of 4)
        if (p.bias_vec4 && kbase + BN <= len_k) {  // warp-uniform
          const float4* b4 = reinterpret_cast<const float4*>(brow + kbase);
#pragma unroll
          for (int c4 = 0; c4 < BN / 4; ++c4) {
            const float4 bv = __ldg(b4 + c4);
            const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
              sr[4 * c4 + u] = __float_as_uint(fmaf(bb[u], kLog2e, __uint_as_float(sr[4 * c4 + u]) * p.scale_log2));
          }
        } else {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            sr[c] = __float_as_uint(
                fmaf(__ldg(brow + min(kbase + c, len_k - 1)), kLog2e, __uint_as_float(sr[c]) * p.scale_log2));
        }
      } else if constexpr (!FAST) {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          float x = __uint_as_float(sr[c]) * p.scale_log2;
          if constexpr (BIAS == kBiasAlibi) x = fmaf(neg_slope2, fabsf(static_cast<float>(kbase + c - i - diag)), x);
          sr[c] = __float_as_uint(x);
        }
      }
      if (edge) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= hi || c < lo) sr[c] = 0xff800000u;  // -inf
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
        mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
      }
      float mx = fmaxf(mx0, mx1);
      if constexpr (FAST) mx *= sc2;  // scale > 0: max commutes with it
      const bool move = mx > m + kRescaleThreshold;
      m_next = move ? mx : m;
      alpha = move ? ex2(m - m_next) : 1.f;
      const float neg_m = m_next == -INFINITY ? 0.f : -m_next;
      // P over the score columns already read: 32 keys -> 16 bf16 pairs per
      // store (P chunk c covers columns [16c, 16c + 16), scores already read).
      // EMU: on tiles with no hidden key (every score finite) one pair in
      // kEmuEvery takes the FMA-pipe exponential instead of the MUFU one.
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = __uint_as_float(sr[c * 32 + 2 * e]), x1 = __uint_as_float(sr[c * 32 + 2 * e + 1]);
          const float a0 = FAST ? fmaf(x0, sc2, neg_m) : x0 + neg_m;
          const float a1 = FAST ? fmaf(x1, sc2, neg_m) : x1 + neg_m;
          float p0, p1;
          // FAST: one pair in kEmuEvery on the FMA pipe.  A hidden key (-inf)
          // then gives about 2^-126 instead of 0: harmless next to a row's
          // largest p (>= 2^-8 under the reference-max rule), and a row with no
          // visible key at all is recognised in the epilogue by m = -inf
          if (FAST && kEmuEvery > 0 && e % (kEmuEvery > 0 ? kEmuEvery : 1) == kEmuEvery - 1) {
            p0 = ex2_poly(a0);
            p1 = ex2_poly(a1);
          } else {
            p0 = ex2(a0);
            p1 = ex2(a1);
          }
          rs0 += p0;
          rs1 += p1;
          pk[e] = pack_bf16(p0, p1);
        }
        tmem_st16(col_s + c * 16, pk);
      }
      l = l * alpha + (rs0 + rs1);
      m = m_next;
      // P_t V of the previous step is complete (its commit preceded this
      // step's scores), so O may be rescaled now
      if (step > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < DV / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(col_o + c * 32, orr);
          tmem_wait_ld();
          reg_fence(orr);
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
          tmem_st32(col_o + c * 32, orr);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.p_full[t]);
    }
    // ---- epilogue: O / l -> bf16 (or fp32 split partial), LSE (natural log)
    if (ok && my.n > 0) ok = __all_sync(0xffffffffu, mbar_wait(&s.o_done[t], 0, ab));
    tc_fence_after();
    if (ok) {
      // a row with no visible key (m never left -inf) is empty
      const bool empty = !(l > 0.f) || m == -INFINITY;
      const float inv_l = empty ? 0.f : 1.f / l;
      __nv_bfloat16* orow = p.o + bidx * p.o_bstride + ((long long)(q_off + i) * p.Hq + h) * DV;
      float* prow = nullptr;
      if constexpr (PARTIAL)
        prow = p.o_part + split * p.part_o_stride + bidx * p.o_bstride + ((long long)(q_off + i) * p.Hq + h) * DV;
#pragma unroll
      for (int c = 0; c < DV / 32; ++c) {
        uint32_t orr[32];
        if (my.n > 0) {
          tmem_ld32(col_o + c * 32, orr);
          tmem_wait_ld();
          reg_fence(orr);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = 0u;
        }
        if constexpr (PARTIAL) {
          if (row_ok) {
            float4* dst = reinterpret_cast<float4*>(prow + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(orr[4 * e]) * inv_l, __uint_as_float(orr[4 * e + 1]) * inv_l,
                                   __uint_as_float(orr[4 * e + 2]) * inv_l, __uint_as_float(orr[4 * e + 3]) * inv_l);
          }
        } else {
          uint32_t packed[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            packed[e] = pack_bf16(__uint_as_float(orr[2 * e]) * inv_l, __uint_as_float(orr[2 * e + 1]) * inv_l);
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
          }
        }
      }
      if (row_ok) {
        const float lse = empty ? -INFINITY : (m + __log2f(l)) * kLn2;
        if constexpr (PARTIAL)
          p.lse_part[split * p.part_lse_stride + bidx * p.lse_bstride + (long long)h * p.lse_hstride + q_off + i] = lse;
        else
          p.lse[bidx * p.lse_bstride + (long long)h * p.lse_hstride + q_off + i] = lse;
      }
    }
  } else {
    if constexpr (kRegSplit) setmaxnreg_dec<kLowRegs>();  // warps 10, 11: idle
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int DV, int BIAS, bool FAST, bool PARTIAL, bool QK8 = false>
int launch_pp_t(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                const FwdParams& p, cudaStream_t st) {
  const size_t smem = sizeof(PPSmem<D, DV, QK8>) + 1024;
  auto kern = fwd_pp_kernel<D, DV, BIAS, FAST, PARTIAL, QK8>;
  if constexpr (kRegSplit) {
    // the split adds up only against a launch of exactly kLaunchRegs a thread
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return ATTN_ERR_CUDA;
    if (fa.numRegs != kLaunchRegs) return ATTN_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const int max_nq = g.cu_q ? g.max_nq : g.Nq;
  const unsigned nblk = (max_nq + 2 * BM - 1) / (2 * BM), nz = (g.cu_q ? g.num_seqs : g.B) * p.num_splits;
  dim3 grid = (!PARTIAL && p.batch_inner) ? dim3(nz, nblk, g.Hq) : dim3(nblk, g.Hq, nz);
  if (grid.y > 65535 || grid.z > 65535) return ATTN_ERR_UNSUPPORTED;
  FwdParams q = p;
  const long long units = (long long)nblk * g.Hq * nz;
  q.grid_nblk = (int)nblk;
  q.grid_nu = g.Hq * (int)nz;
  q.half_from = (int)std::min<long long>(units, INT_MAX);
  // Equal units (no causal mask, no window, dense batches) in one CTA per SM:
  // when the last wave would fill at most half the SMs, its units run as single
  // 128-row tiles, two CTAs each, and the wave ends sooner.
  if (!PARTIAL && !p.batch_inner && !g.cu_q && !g.causal && g.window_left < 0 && g.window_right < 0) {
    const long long sms = sm_count(), tail = units % sms;
    if (units >= sms && tail > 0 && 2 * tail <= sms && units + tail < INT_MAX) {
      q.half_from = (int)(units - tail);
      grid = dim3((unsigned)(units + tail));
    }
  }
  record_kernel_event(ATTN_KERNEL_FWD, 0, st);
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, q);
  record_kernel_event(ATTN_KERNEL_FWD, 1, st);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Head widths (D, DV) and bias kinds instantiated for one width pair.
template <int D, int DV>
int dispatch_pp(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                const FwdParams& p, int bias_kind, bool fast, bool partial, cudaStream_t st) {
  if (partial) {  // split partials: no bias
    if (bias_kind != kBiasNone) return ATTN_ERR_UNSUPPORTED;
    return fast ? launch_pp_t<D, DV, kBiasNone, true, true>(g, mq, mk, mv, p, st)
                : launch_pp_t<D, DV, kBiasNone, false, true>(g, mq, mk, mv, p, st);
  }
  if constexpr (D == DV) {
    if (bias_kind == kBiasDense) return launch_pp_t<D, DV, kBiasDense, false, false>(g, mq, mk, mv, p, st);
    if (bias_kind == kBiasAlibi) return launch_pp_t<D, DV, kBiasAlibi, false, false>(g, mq, mk, mv, p, st);
  } else {
    if (bias_kind != kBiasNone) return ATTN_ERR_UNSUPPORTED;
  }
  return fast ? launch_pp_t<D, DV, kBiasNone, true, false>(g, mq, mk, mv, p, st)
              : launch_pp_t<D, DV, kBiasNone, false, false>(g, mq, mk, mv, p, st);
}

}  // namespace

int launch_fwd_pp_fp8(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const FwdParams& p, cudaStream_t st) {
  if (g.D != 128 || (g.Dv && g.Dv != 128) || g.cu_q || g.bias || g.alibi || !(g.scale > 0.f))
    return ATTN_ERR_UNSUPPORTED;
  return launch_pp_t<128, 128, kBiasNone, true, false, true>(g, mq, mk, mv, p, st);
}

int launch_fwd_pp(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const FwdParams& p, int bias_kind, bool fast, bool partial, cudaStream_t st) {
  const int dv = g.Dv ? g.Dv : g.D;
  if (g.D == 128 && dv == 128) return dispatch_pp<128, 128>(g, mq, mk, mv, p, bias_kind, fast, partial, st);
  if (g.D == 64 && dv == 64) return dispatch_pp<64, 64>(g, mq, mk, mv, p, bias_kind, fast, partial, st);
  if (partial) return ATTN_ERR_UNSUPPORTED;
  if (g.D == 128 && dv == 64) return dispatch_pp<128, 64>(g, mq, mk, mv, p, bias_kind, fast, false, st);
  if (g.D == 64 && dv == 128) return dispatch_pp<64, 128>(g, mq, mk, mv, p, bias_kind, fast, false, st);
  return ATTN_ERR_UNSUPPORTED;
}

}  // namespace attn
