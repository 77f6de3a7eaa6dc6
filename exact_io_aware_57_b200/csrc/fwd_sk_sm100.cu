// Forward attention on sm_100a tensor cores: one 128-row query tile per CTA,
// its softmax split over the keys between two warpgroups.
//
// The CTA streams 128-key tiles of K and V past its query tile ("Attention IO
// tiling" lesson card, The mechanism: tiles staged on chip, each score block
// folded into the per-row softmax state and then dropped).  The exponentials
// of a 128 x 128 score tile are the slow part of a step, so two warpgroups
// share every row: thread r of warpgroup h owns query row r and keys
// [64h, 64h + 64) of each tile.  They agree on the row's reference max through
// shared memory once per tile and keep partial row sums that add up at the end
// (the same (m, l, a) state of "Softmax does not need the matrix", "Carry the
// Normalizer", split by keys: l = l_0 + l_1 for a common m).
//
//   warp 0      TMA producer: Q once, then K_j / V_j into a 3- or 4-stage smem ring
//   warp 1      TMEM owner + single-thread tcgen05.mma issuer
//   warps 2..5  softmax, keys [0, 64) of each tile: thread r owns row r (TMEM lane r)
//   warps 6..9  softmax, keys [64, 128) of each tile
//
// TMEM (512 columns x 128 lanes x 32 bit):
//   [  0,128) S buffer 0   [128,256) S buffer 1     (fp32 scores, S = Q K_j^T)
//   [256,256+DV) O accumulator (fp32)
//   [384,448) P buffer 0   [448,512) P buffer 1     (bf16 pairs, A operand of P V_j)
// S and P are double-buffered: S_{j+2} is computed while the softmax works on
// S_j, interleaved with P_j V_j on the tensor pipe.
//
// Per key tile the softmax thread forms x = s * scale * log2(e) (+ bias *
// log2(e)), the row max over both halves, moves its reference max m only when
// the tile max exceeds it by more than 2^8 (O / l and LSE do not depend on the
// reference), p = 2^(x - m), l_h = 2^(m_old - m) l_h + sum of its p, writes its
// half of P and -- once P_{j-1} V_{j-1} has landed -- rescales its half of the
// O row by 2^(m_old - m) when m moved.  After the last tile O / (l_0 + l_1)
// and LSE = (m + log2(l_0 + l_1)) ln 2 are written.
// Causal and local attention load only the key tiles meeting the visible band
// and mask only the tiles on its edges ("Understanding FlashAttention Pt 1",
// contents 3.5 and 4.2).  Split-KV: with num_splits > 1 the grid's z index
// also runs over key ranges, each CTA writing O_t (fp32) and LSE_t for the
// merge.  QK8: Q and K are e4m3 (FP8 forward; S on the e4m3 tensor cores and
// rescaled by the per-head quantisation scales, P V in bf16).
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace attn {

namespace {

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 128;  // keys per KV tile
constexpr int KH = BN / 2;  // keys per softmax thread and tile
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
constexpr float kRescaleThreshold = 8.f;  // log2 units: P stays <= 256
#ifndef ATTN_EX2_EMU_EVERY
#define ATTN_EX2_EMU_EVERY 0
#endif
// One bf16 pair of P in kEmuEvery is exponentiated on the FMA pipe (0: none).
constexpr int kEmuEvery = ATTN_EX2_EMU_EVERY;

// K/V stages: as many as fit beside the Q tile and 3 KB of barriers and
// exchange slots in 227 KB (at most four).
template <int D, int DV, bool QK8>
constexpr int kStages = ((227 - 3) * 1024 - BM * D * (QK8 ? 1 : 2)) / (BN * D * (QK8 ? 1 : 2) + BN * DV * 2) < 4
                            ? ((227 - 3) * 1024 - BM * D * (QK8 ? 1 : 2)) / (BN * D * (QK8 ? 1 : 2) + BN * DV * 2)
                            : 4;

template <int D, int DV, bool QK8>
struct SkSmem {
  static constexpr int NST = kStages<D, DV, QK8>;
  static constexpr int kQKBytes = BM * D * (QK8 ? 1 : 2);  // Q or K tile
  static constexpr int kVBytes = BN * DV * 2;
  alignas(1024) uint8_t q[kQKBytes];
  alignas(1024) uint8_t k[NST][kQKBytes];
  alignas(1024) uint8_t v[NST][kVBytes];
  // [step parity][key half][row]: tile row maxima exchanged by the halves; after
  // the last step the slot of the other parity carries the partial row sums
  float mx[2][2][BM];
  uint64_t q_full;
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_done, mx_ready, l_ready, drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int N>
ATTN_DEVINL void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// 10 warps: three of them share one SM sub-partition's 16K registers, so a
// thread gets at most 168.
template <int D, int DV, int BIAS, bool FAST, bool PARTIAL, bool QK8 = false>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Smem = SkSmem<D, DV, QK8>;
  constexpr int NST = Smem::NST;
  constexpr int KB = D * (QK8 ? 1 : 2) / 128;  // 128-byte blocks per Q/K row
  constexpr int kBoxCols = QK8 ? 128 : 64;     // elements in one 128-byte block
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the swizzle needs 1024-byte aligned tiles
    if (threadIdx.x == 0) atomicExch(p.status, ATTN_ERR_CUDA);
    return;
  }

  // ---- work tile: heavy (late) query tiles first under causal masking
  const int m_tile = p.causal ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
  const int h = blockIdx.y;
  const int z = PARTIAL ? (int)blockIdx.z / p.num_splits : (int)blockIdx.z;
  const int split = PARTIAL ? (int)blockIdx.z % p.num_splits : 0;
  int q_off = 0, len_q = p.Nq, k_off = 0, len_k = p.Nk, bidx = z;
  if (p.cu_q) {
    // invalid offsets: reported in the status word, nothing read or written
    if (!packed_seq(p.cu_q, z, p.Nq, p.max_nq, p.status, q_off, len_q) ||
        !packed_seq(p.cu_k, z, p.Nk, p.max_nk, p.status, k_off, len_k))
      return;
    bidx = 0;
  }
  const int m0 = m_tile * BM;
  if (m0 >= len_q) return;  // uniform: before any barrier or TMEM use
  const int hk = h / (p.Hq / p.Hkv);
  const int diag = len_k - len_q;  // row i is aligned with key i + diag
  // keys [kv_begin, kv_end) hold every key visible from rows m0 .. m0 + BM - 1,
  // clipped to this CTA's split of the keys (|m0|, |diag| < 2^28, win_* <= 2^30)
  const int rows_end = min(m0 + BM, len_q);
  const int kv_end = min(PARTIAL ? min(len_k, (split + 1) * p.split_len) : len_k, rows_end + diag + p.win_r);
  const int kv_begin = max(PARTIAL ? split * p.split_len : 0, m0 + diag - p.win_l);
  const int j_first = kv_begin / BN;
  const int n_kv = kv_end > kv_begin ? (kv_end + BN - 1) / BN - j_first : 0;

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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i], 8);
    }
    mbar_init(&s.pv_done, 1);
    mbar_init(&s.o_done, 1);
    mbar_init(&s.mx_ready, 8);
    mbar_init(&s.l_ready, 8);
    mbar_init(&s.drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const Abort ab{&s.abort_flag, p.status, p.wait_limit};

  if (warp == 0) {
    // ===================================================== TMA producer
    // no visible tile: load nothing (no copy may be left in flight at exit)
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_expect_tx(&s.q_full, Smem::kQKBytes);
#pragma unroll
      for (int kb = 0; kb < KB; ++kb)
        tma_load_4d(s.q + kb * BM * 128, &tm_q, &s.q_full, kb * kBoxCols, h, q_off + m0, bidx);
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % NST;
        const uint32_t ph = (j / NST) & 1;
        const int row = k_off + (j_first + j) * BN;
        if (!mbar_wait(&s.k_empty[st], ph ^ 1, ab)) break;
        mbar_expect_tx(&s.k_full[st], Smem::kQKBytes);
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
        for (int j = max(0, issued_k - NST); j < issued_k; ++j)
          mbar_wait_drain(&s.k_full[j % NST], (j / NST) & 1, p.wait_limit);
        for (int j = max(0, issued_v - NST); j < issued_v; ++j)
          mbar_wait_drain(&s.v_full[j % NST], (j / NST) & 1, p.wait_limit);
      }
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t idesc_pv = idesc_bf16(BM, DV, 0, 1);  // P: TMEM, V_j: MN-major
      const uint32_t q_addr = smem_u32(s.q);
      // S_j = Q K_j^T into S buffer j & 1: one instruction per 32 bytes of the
      // rows (K = 16 bf16 or 32 e4m3 elements)
      auto s_mma = [&](int j, int kk) {
        const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
        const uint32_t k_addr = smem_u32(s.k[j % NST]);
        if constexpr (QK8)
          mma_ss_f8(tmem + kColS + (j & 1) * BN, sdesc_sw128(q_addr + off, 16, 1024),
                    sdesc_sw128(k_addr + off, 16, 1024), idesc_e4m3(BM, BN), kk > 0);
        else
          mma_ss(tmem + kColS + (j & 1) * BN, sdesc_sw128(q_addr + off, 16, 1024),
                 sdesc_sw128(k_addr + off, 16, 1024), idesc_bf16(BM, BN, 0, 0), kk > 0);
      };
      auto issue_s = [&](int j) -> bool {
        const int st = j % NST;
        if (!mbar_wait(&s.k_full[st], (j / NST) & 1, ab)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < KB * 4; ++kk) s_mma(j, kk);
        mma_commit(&s.s_full[j & 1]);
        mma_commit(&s.k_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&s.q_full, 0, ab);
      if (ok) ok = issue_s(0);
      if (ok && n_kv > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int buf = j & 1, st = j % NST;
        // p_full(j): P_j is in TMEM, O is rescaled, and S buffer `buf` has been read
        if (!mbar_wait(&s.p_full[buf], (j >> 1) & 1, ab)) break;
        if (!mbar_wait(&s.v_full[st], (j / NST) & 1, ab)) break;
        const bool next = j + 2 < n_kv;
        if (next && !mbar_wait(&s.k_full[(j + 2) % NST], ((j + 2) / NST) & 1, ab)) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(s.v[st]);
        // O += P_j V_j interleaved with S_{j+2} = Q K_{j+2}^T: two independent
        // accumulators keep the tensor pipe streaming
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ts(tmem + kColO, tmem + kColP + buf * 64 + kk * 8, sdesc_sw128(v_addr + kk * 2048, BN * 128, 1024),
                 idesc_pv, (j > 0 || kk > 0));
          if (next && kk < KB * 4) s_mma(j + 2, kk);
        }
        mma_commit(&s.pv_done);
        mma_commit(&s.v_empty[st]);
        if (next) {
          mma_commit(&s.s_full[buf]);
          mma_commit(&s.k_empty[(j + 2) % NST]);
        }
      }
      // the epilogue's signal: every P V is done (pv_done alone cannot say so,
      // the softmax does not wait on each of its phases)
      if (ok) mma_commit(&s.o_done);
      // TMEM must be quiescent before it is released
      mma_commit(&s.drain);
      mbar_wait_drain(&s.drain, 0, p.wait_limit);
    }
  } else {
    // ===================================================== softmax warpgroups
    const int khalf = (warp - 2) >> 2;  // keys [64 khalf, 64 khalf + 64) of each tile
    const int quarter = warp & 3;       // TMEM lanes [32 quarter, 32 quarter + 32)
    const int r = quarter * 32 + lane;
    const int i = m0 + r;  // row inside its sequence
    const bool row_ok = i < len_q;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float* brow = nullptr;  // rows past the end read the last row (their output is dropped)
    if constexpr (BIAS == kBiasDense)
      brow = p.bias + bidx * p.bias_bstride + ((long long)h * p.Nq + min(i, len_q - 1)) * p.Nk;
    float neg_slope2 = 0.f;  // ALiBi: B = -slope |key - (i + diag)|, in log2 units
    if constexpr (BIAS == kBiasAlibi) neg_slope2 = -__ldg(p.alibi + h) * kLog2e;
    // log2(e) * scale, times the e4m3 scales of this (batch, head) of Q and K in the FP8 forward
    float sc2 = p.scale_log2;
    if constexpr (QK8) sc2 *= __ldg(p.q_scale + bidx * p.Hq + h) * __ldg(p.k_scale + bidx * p.Hkv + hk);
    // m: the reference max of the row (log2 units), common to both halves; l:
    // this half's share of the row sum against m
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int buf = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s.s_full[buf], (j >> 1) & 1, ab));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[KH];
      tmem_ld32(tmem + lane_off + kColS + buf * BN + khalf * KH, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tmem + lane_off + kColS + buf * BN + khalf * KH + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      reg_fence(sr);
      const int ktile = (j_first + j) * BN;  // first key of the tile
      const int kbase = ktile + khalf * KH;  // first key of this half
      if constexpr (!FAST) {
        // general scores: x = s * scale * log2(e) (+ bias * log2(e))
#pragma unroll
        for (int c = 0; c < KH; ++c) {
          float x = __uint_as_float(sr[c]) * p.scale_log2;
          if constexpr (BIAS == kBiasDense) x = fmaf(__ldg(brow + min(kbase + c, len_k - 1)), kLog2e, x);
          if constexpr (BIAS == kBiasAlibi) x = fmaf(neg_slope2, fabsf(static_cast<float>(kbase + c - i - diag)), x);
          sr[c] = __float_as_uint(x);
        }
      }
      // tile on an edge of the visible band, or ragged: keys outside [lo, hi) of this half are hidden
      const bool edge =
          (ktile + BN > len_k) || (ktile + BN - 1 > m0 + diag + p.win_r) || (ktile < m0 + BM - 1 + diag - p.win_l);
      if (edge) {
        const int hi = min(len_k, i + diag + p.win_r + 1) - kbase;
        const int lo = i + diag - p.win_l - kbase;
#pragma unroll
        for (int c = 0; c < KH; ++c)
          if (c >= hi || c < lo) sr[c] = 0xff800000u;  // -inf
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int c = 0; c < KH; c += 2) {
        mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
        mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
      }
      // the row max over both halves: each half posts its own, then reads the other's
      s.mx[buf][khalf][r] = fmaxf(mx0, mx1);
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.mx_ready);
      ok = __all_sync(0xffffffffu, mbar_wait(&s.mx_ready, j & 1, ab));
      if (!ok) break;
      float mx = fmaxf(s.mx[buf][0][r], s.mx[buf][1][r]);
      if constexpr (FAST) mx *= sc2;  // scale > 0: max commutes with it
      const bool move = mx > m + kRescaleThreshold;
      const float m_next = move ? mx : m;
      const float alpha = move ? ex2(m - m_next) : 1.f;
      const float neg_m = m_next == -INFINITY ? 0.f : -m_next;
      float rs0 = 0.f, rs1 = 0.f;
      // this half of P (64 keys -> 32 bf16 pairs, columns [32 khalf, 32 khalf + 32)
      // of P buffer `buf`, free since S_j's commit also covered P_{j-2} V_{j-2}).
      // EMU: on tiles with no hidden key one pair in kEmuEvery is exponentiated
      // on the FMA pipe instead of the MUFU.
      auto exps = [&](auto emu) {
        constexpr bool EMU = decltype(emu)::value;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = __uint_as_float(sr[c * 32 + 2 * e]), x1 = __uint_as_float(sr[c * 32 + 2 * e + 1]);
            const float a0 = FAST ? fmaf(x0, sc2, neg_m) : x0 + neg_m;
            const float a1 = FAST ? fmaf(x1, sc2, neg_m) : x1 + neg_m;
            float p0, p1;
            if (EMU && e % kEmuEvery == kEmuEvery - 1) {
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
          tmem_st16(tmem + lane_off + kColP + buf * 64 + khalf * 32 + c * 16, pk);
        }
      };
      if constexpr (kEmuEvery > 0) {
        if (!edge)
          exps(std::true_type{});
        else
          exps(std::false_type{});
      } else {
        exps(std::false_type{});
      }
      l = l * alpha + (rs0 + rs1);
      m = m_next;
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // this half of the O row, once P_{j-1} V_{j-1} has landed.  The commit of
        // S_j covered P_{j-2} V_{j-2}, so pv_done is at most one phase behind
        // phase j-1 here and its parity names the phase unambiguously
        ok = __all_sync(0xffffffffu, mbar_wait(&s.pv_done, (j - 1) & 1, ab));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < DV / 64; ++c) {
          uint32_t orr[32];
          const uint32_t col = tmem + lane_off + kColO + khalf * (DV / 2) + c * 32;
          tmem_ld32(col, orr);
          tmem_wait_ld();
          reg_fence(orr);
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
          tmem_st32(col, orr);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.p_full[buf]);
    }
    // ---- epilogue: l = l_0 + l_1; this half of O / l -> bf16 (or fp32 split
    // partial); LSE (natural log) from the first half
    // every warp read the maxima of step n_kv - 2 before arriving at step n_kv - 1:
    // that slot is free for the partial sums
    float(&lsum)[2][BM] = s.mx[n_kv & 1];
    if (ok) {
      lsum[khalf][r] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.l_ready);
      ok = __all_sync(0xffffffffu, mbar_wait(&s.l_ready, 0, ab));
    }
    if (ok && n_kv > 0) ok = __all_sync(0xffffffffu, mbar_wait(&s.o_done, 0, ab));
    tc_fence_after();
    if (ok) {
      const float lt = lsum[0][r] + lsum[1][r];
      const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
      const int c0 = khalf * (DV / 2);  // first O column of this half
      __nv_bfloat16* orow = p.o + bidx * p.o_bstride + ((long long)(q_off + i) * p.Hq + h) * DV + c0;
      float* prow = nullptr;
      if constexpr (PARTIAL)
        prow = p.o_part + split * p.part_o_stride + bidx * p.o_bstride + ((long long)(q_off + i) * p.Hq + h) * DV + c0;
#pragma unroll
      for (int c = 0; c < DV / 64; ++c) {
        uint32_t orr[32];
        if (n_kv > 0) {
          tmem_ld32(tmem + lane_off + kColO + c0 + c * 32, orr);
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
      if (row_ok && khalf == 0) {
        const float lse = lt > 0.f ? (m + __log2f(lt)) * kLn2 : -INFINITY;
        if constexpr (PARTIAL)
          p.lse_part[split * p.part_lse_stride + bidx * p.lse_bstride + (long long)h * p.lse_hstride + q_off + i] = lse;
        else
          p.lse[bidx * p.lse_bstride + (long long)h * p.lse_hstride + q_off + i] = lse;
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int DV, int BIAS, bool FAST, bool PARTIAL, bool QK8 = false>
int launch_sk_t(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                const FwdParams& p, cudaStream_t st) {
  // at least half of the SM's shared memory, so that a second CTA never waits
  // on the 512 TMEM columns this one holds (227 KB at most: checked at compile time)
  static_assert(sizeof(SkSmem<D, DV, QK8>) <= 227 * 1024, "shared memory");
  const size_t smem = std::max<size_t>(sizeof(SkSmem<D, DV, QK8>), 116 * 1024);
  auto kern = fwd_sk_kernel<D, DV, BIAS, FAST, PARTIAL, QK8>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const int max_nq = g.cu_q ? g.max_nq : g.Nq;
  dim3 grid((max_nq + BM - 1) / BM, g.Hq, (g.cu_q ? g.num_seqs : g.B) * p.num_splits);
  record_kernel_event(ATTN_KERNEL_FWD, 0, st);
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, p);
  record_kernel_event(ATTN_KERNEL_FWD, 1, st);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, int DV>
int dispatch_sk(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                const FwdParams& p, int bias_kind, bool fast, bool partial, cudaStream_t st) {
  if (partial) {  // split partials: no bias
    if (bias_kind != kBiasNone) return ATTN_ERR_UNSUPPORTED;
    return fast ? launch_sk_t<D, DV, kBiasNone, true, true>(g, mq, mk, mv, p, st)
                : launch_sk_t<D, DV, kBiasNone, false, true>(g, mq, mk, mv, p, st);
  }
  if constexpr (D == DV) {
    if (bias_kind == kBiasDense) return launch_sk_t<D, DV, kBiasDense, false, false>(g, mq, mk, mv, p, st);
    if (bias_kind == kBiasAlibi) return launch_sk_t<D, DV, kBiasAlibi, false, false>(g, mq, mk, mv, p, st);
  } else {
    if (bias_kind != kBiasNone) return ATTN_ERR_UNSUPPORTED;
  }
  return fast ? launch_sk_t<D, DV, kBiasNone, true, false>(g, mq, mk, mv, p, st)
              : launch_sk_t<D, DV, kBiasNone, false, false>(g, mq, mk, mv, p, st);
}

}  // namespace

int launch_fwd_sk(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const FwdParams& p, int bias_kind, bool fast, bool partial, cudaStream_t st) {
  const int dv = g.Dv ? g.Dv : g.D;
  if (g.D == 128 && dv == 128) return dispatch_sk<128, 128>(g, mq, mk, mv, p, bias_kind, fast, partial, st);
  if (g.D == 64 && dv == 64) return dispatch_sk<64, 64>(g, mq, mk, mv, p, bias_kind, fast, partial, st);
  if (partial) return ATTN_ERR_UNSUPPORTED;
  if (g.D == 128 && dv == 64) return dispatch_sk<128, 64>(g, mq, mk, mv, p, bias_kind, fast, false, st);
  if (g.D == 64 && dv == 128) return dispatch_sk<64, 128>(g, mq, mk, mv, p, bias_kind, fast, false, st);
  return ATTN_ERR_UNSUPPORTED;
}

int launch_fwd_sk_fp8(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const FwdParams& p, cudaStream_t st) {
  if (g.D != 128 || (g.Dv && g.Dv != 128) || g.cu_q || g.bias || g.alibi || !(g.scale > 0.f))
    return ATTN_ERR_UNSUPPORTED;
  return launch_sk_t<128, 128, kBiasNone, true, false, true>(g, mq, mk, mv, p, st);
}

}  // namespace attn
