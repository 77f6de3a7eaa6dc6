// Forward attention with a dense additive bias on sm_100a tensor cores: two
// query tiles per CTA and 64-key tiles with double-buffered scores.
//
// One CTA owns 256 query rows of one (batch, head), as two tiles of 128 rows,
// and streams 64-key tiles of K and V past both ("Attention IO tiling" lesson
// card, The mechanism: tiles staged on chip, each score block folded into the
// per-row softmax state and then dropped).  With 64-key tiles each query
// tile's scores take 64 TMEM columns, so every tile has two score buffers: the
// scores of the next key tile are ready while the softmax reads its bias rows
// and works on the current one ("Understanding FlashAttention Pt 1", contents
// 5.5: overlap data movement, matrix products and the softmax).  Measured on
// the grouped causal workload with its 2.1 GB fp32 bias this runs the forward
// at about twice the speed of the 128-key two-tile kernel; without a bias
// tensor to read, the 128-key kernel is faster and is used instead.
//
//   warps 0..3  softmax of query tile 0: thread r owns query row r (TMEM lane r)
//   warps 4..7  softmax of query tile 1
//   warp 8      TMEM owner + single-thread tcgen05.mma issuer
//   warp 9      TMA producer: Q_0, Q_1 once, then K_j (two key tiles ahead) and
//               V_j into smem rings
//   warp 10     (BT: bias rows 16-byte aligned) TMA producer of the bias: each
//               query tile's 128 x 64 fp32 bias block of its next key tile, into
//               a buffer of its own that the softmax empties first thing, so the
//               block of the next key tile is on its way while the softmax works
//
// TMEM (512 columns x 128 lanes x 32 bit):
//   [128 t + 64 b, 128 t + 64 b + 64)  S_t of the key tiles with step parity b
//                                      (fp32); P_t (bf16 pairs) over its first 32
//   [256 + D t, 256 + D t + D)         O_t (fp32 accumulator)
//
// MMA issue order per key tile j (each query tile only where j is in its range):
//   O_0 += P_0 V_j;  S_0 = Q_0 K_{j+2}^T;  O_1 += P_1 V_j;  S_1 = Q_1 K_{j+2}^T
// S of key tile j + 2 takes the buffer that P of key tile j leaves; tcgen05.mma
// executes in issue order, so P_t V_j has read P before the scores overwrite it.
//
// Per key tile the softmax thread of row i forms x = (s * scale + bias) *
// log2(e), moves its reference max m only when the tile max exceeds m by more
// than 2^8 (the final O / l and LSE do not depend on the reference),
// p = 2^(x - m), l = 2^(m_old - m) l + sum p ("Softmax does not need the
// matrix", "Carry the Normalizer", in base 2), writes P over the scores it has
// read and hands the tile to the MMA warp.  When m moves it rescales its O row
// by 2^(m_old - m), after the previous key tile's P V has completed: the scores
// of the next key tile were issued after that P V, so their completion (or, for
// a tile's last key tile, a commit of its own) tells.  After the last key tile
// it writes O / l and LSE = (m + log2 l) ln 2.  Causal and local masks apply
// to the key tiles on the edges of a query tile's band only.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace attn {

namespace {

constexpr int BM = 128;  // query rows per tile (two tiles per CTA)
constexpr int KT = 64;   // keys per K/V tile
constexpr int kWarpMma = 8, kWarpLoad = 9, kWarpBias = 10;
template <bool BT>
constexpr int kThreadsOf = BT ? 352 : 320;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.f;  // log2 units: P stays <= 256

// BT: each query tile's bias block (128 rows x 64 keys fp32, two 128B-swizzled
// TMA boxes of 32 keys) is staged in shared memory.
template <int D, bool BT>
struct DBSmem {
  static constexpr int DV = D;
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kKBytes = KT * D * 2;
  static constexpr int kVBytes = KT * DV * 2;
  static constexpr int kBiasBytes = BM * KT * 4;  // one query tile's block
  // K/V ring depth: as many stages as fit beside the two Q tiles (and the two
  // bias blocks) in ~222 KB (~226 KB with the bias blocks)
  static constexpr int NST =
      std::min(8, ((BT ? 226 : 222) * 1024 - 2 * kQBytes - (BT ? 2 * kBiasBytes : 0)) / (kKBytes + kVBytes));
  alignas(1024) uint8_t q[2][kQBytes];
  alignas(1024) uint8_t k[NST][kKBytes];
  alignas(1024) uint8_t v[NST][kVBytes];
  alignas(1024) uint8_t bias[2][BT ? kBiasBytes : 16];
  uint64_t q_full;
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full[2][2], p_full[2][2];  // [query tile][score buffer]
  uint64_t bias_full[2], bias_empty[2];  // BT: [query tile]
  uint64_t pv_last[2], o_done[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int N>
ATTN_DEVINL void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// Key-tile range of one query tile: 64-key tiles jb .. jb + n - 1 hold every
// key visible from its rows [mt, min(mt + BM, len_q)), clipped to [k_lo, k_hi).
struct TileRange {
  int jb, n;
};

ATTN_DEVINL TileRange tile_range(int mt, int len_q, int diag, int win_l, int win_r, int k_lo, int k_hi) {
  TileRange r{0, 0};
  if (mt >= len_q) return r;
  const int rows_end = min(mt + BM, len_q);
  const int kv_end = min(k_hi, rows_end + diag + win_r);
  const int kv_begin = max(k_lo, mt + diag - win_l);
  if (kv_end <= kv_begin) return r;
  r.jb = kv_begin / KT;
  r.n = (kv_end + KT - 1) / KT - r.jb;
  return r;
}

ATTN_DEVINL bool in_range(const TileRange& r, int j) { return r.n > 0 && j >= r.jb && j < r.jb + r.n; }

template <int D, bool BT>
__global__ void __launch_bounds__(kThreadsOf<BT>, 1)
    fwd_db_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_b,
                  const FwdParams p) {
  using Smem = DBSmem<D, BT>;
  constexpr int DV = D;
  constexpr int NST = Smem::NST;
  constexpr int KB = D / 64, KBV = DV / 64;  // 128-byte blocks per Q/K and V row
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work: heavy (late) row blocks first under causal masking, the row
  // blocks of a group of (batch, head) pairs interleaved (grouped_unit): eight
  // heads of one batch element, or, when the batch elements share the bias
  // (grid (batch, row block, head)), every batch element of two heads, so that
  // the ones reading the same bias rows run side by side
  const bool bi = p.batch_inner;
  const int nblk = bi ? (int)gridDim.y : (int)gridDim.x, nb = bi ? (int)gridDim.x : (int)gridDim.z;
  int blk_raw, u;
  grouped_unit(nblk, nb * p.Hq, bi ? 2 * nb : 8, blk_raw, u);
  const int blk = p.causal ? nblk - 1 - blk_raw : blk_raw;
  const int h = bi ? u / nb : u % p.Hq;
  const int bidx = bi ? u % nb : u / p.Hq;
  const int q_off = 0, k_off = 0, len_q = p.Nq, len_k = p.Nk;
  const int m0 = blk * 2 * BM;
  if (m0 >= len_q) return;  // uniform: before any barrier or TMEM use
  const int hk = h / (p.Hq / p.Hkv);
  const int diag = len_k - len_q;  // row i is aligned with key i + diag
  const int k_lo = 0, k_hi = len_k;
  TileRange rg[2];
  rg[0] = tile_range(m0, len_q, diag, p.win_l, p.win_r, k_lo, k_hi);
  rg[1] = tile_range(m0 + BM, len_q, diag, p.win_l, p.win_r, k_lo, k_hi);
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
      for (int b = 0; b < 2; ++b) {
        mbar_init(&s.s_full[t][b], 1);
        mbar_init(&s.p_full[t][b], 4);
      }
      mbar_init(&s.pv_last[t], 1);
      mbar_init(&s.o_done[t], 1);
      mbar_init(&s.bias_full[t], 1);
      mbar_init(&s.bias_empty[t], 4);  // the four warps of the tile's softmax
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
          tma_load_4d(s.q[t] + kb * BM * 128, &tm_q, &s.q_full, kb * 64, h, q_off + m0 + t * BM, bidx);
      }
      // K runs two key tiles ahead of V, as the scores run two key tiles ahead
      // of P V: each ring then keeps its full depth of loads in flight
      int issued_k = 0, issued_v = 0;
      for (int i = 0; i < n_union + 2; ++i) {
        if (i < n_union) {
          const int st = i % NST;
          if (!mbar_wait(&s.k_empty[st], ((i / NST) & 1) ^ 1, ab)) break;
          mbar_expect_tx(&s.k_full[st], Smem::kKBytes);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            tma_load_4d(s.k[st] + kb * KT * 128, &tm_k, &s.k_full[st], kb * 64, hk, k_off + (J0 + i) * KT, bidx);
          ++issued_k;
        }
        if (i >= 2) {
          const int iv = i - 2, st = iv % NST;
          if (!mbar_wait(&s.v_empty[st], ((iv / NST) & 1) ^ 1, ab)) break;
          mbar_expect_tx(&s.v_full[st], Smem::kVBytes);
#pragma unroll
          for (int kb = 0; kb < KBV; ++kb)
            tma_load_4d(s.v[st] + kb * KT * 128, &tm_v, &s.v_full[st], kb * 64, hk, k_off + (J0 + iv) * KT, bidx);
          ++issued_v;
        }
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
  } else if (BT && warp == kWarpBias) {
    // ===================================================== bias producer
    // One buffer per query tile: the block of its key tile `step` is loaded once
    // the softmax has read the block of step - 1 out of shared memory.
    if (lane == 0 && n_union > 0) {
      tma_prefetch_desc(&tm_b);
      const int row = q_off + m0, zb = p.bias_bstride ? bidx : 0;
      int issued[2] = {0, 0};
      bool ok = true;
      for (int step = 0; ok && step < max(rg[0].n, rg[1].n); ++step) {
        for (int t = 0; t < 2; ++t) {
          if (step >= rg[t].n) continue;
          if (step > 0 && !(ok = mbar_wait(&s.bias_empty[t], (step - 1) & 1, ab))) break;
          mbar_expect_tx(&s.bias_full[t], Smem::kBiasBytes);
          const int kb = k_off + (rg[t].jb + step) * KT;  // a multiple of 64 keys: 16-byte aligned
#pragma unroll
          for (int half = 0; half < 2; ++half)
            tma_load_4d(s.bias[t] + half * (BM * 128), &tm_b, &s.bias_full[t], kb + 32 * half, row + t * BM, h, zb);
          ++issued[t];
        }
      }
      if (s.abort_flag) {
        // at most one block per buffer is in flight: the last one issued
        for (int t = 0; t < 2; ++t)
          if (issued[t] > 0) mbar_wait_drain(&s.bias_full[t], (issued[t] - 1) & 1, p.wait_limit);
      }
    }
  } else if (warp == kWarpMma) {
    // ===================================================== MMA issuer
    if (lane == 0 && n_union > 0) {
      constexpr uint32_t idesc_s = idesc_bf16(BM, KT, 0, 0);   // Q_t: K-major, K_j: K-major
      constexpr uint32_t idesc_pv = idesc_bf16(BM, DV, 0, 1);  // P_t: TMEM, V_j: MN-major
      // S_t(j) = Q_t K_j^T into the buffer of its step parity.  K_j is released
      // once its last user has been issued (tile 0's S of a key tile always
      // precedes tile 1's).
      auto issue_s = [&](int t, int j) -> bool {
        const int i = j - J0, st = i % NST;
        if (!mbar_wait(&s.k_full[st], (i / NST) & 1, ab)) return false;
        tc_fence_after();
        const int b = (j - rg[t].jb) & 1;
        const uint32_t q_addr = smem_u32(s.q[t]), k_addr = smem_u32(s.k[st]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + t * 128 + b * 64, sdesc_sw128(q_addr + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(k_addr + (kk >> 2) * (KT * 128) + (kk & 3) * 32, 16, 1024), idesc_s, kk > 0);
        mma_commit(&s.s_full[t][b]);
        if (t == 1 || !in_range(rg[1], j)) mma_commit(&s.k_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&s.q_full, 0, ab);
      // the first two key tiles of each query tile's range that start here
      for (int j = J0; ok && j < J0 + 2; ++j)
        for (int t = 0; ok && t < 2; ++t)
          if (in_range(rg[t], j)) ok = issue_s(t, j);
      for (int j = J0; ok && j < J1; ++j) {
        const int i = j - J0, st = i % NST;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok) break;
          if (in_range(rg[t], j)) {
            const int step = j - rg[t].jb;
            if (!(ok = mbar_wait(&s.p_full[t][step & 1], (step >> 1) & 1, ab))) break;
            if (!(ok = mbar_wait(&s.v_full[st], (i / NST) & 1, ab))) break;
            tc_fence_after();
            const uint32_t v_addr = smem_u32(s.v[st]);
            // O_t += P_t V_j (P_t from TMEM over the first 32 columns of its scores)
#pragma unroll
            for (int kk = 0; kk < KT / 16; ++kk)
              mma_ts(tmem + 256 + t * DV, tmem + t * 128 + (step & 1) * 64 + kk * 8,
                     sdesc_sw128(v_addr + kk * 2048, KT * 128, 1024), idesc_pv, (step > 0 || kk > 0));
            if (t == 1 || !in_range(rg[1], j)) mma_commit(&s.v_empty[st]);
            if (step == rg[t].n - 2) mma_commit(&s.pv_last[t]);
            if (step == rg[t].n - 1) mma_commit(&s.o_done[t]);
          }
          // the scores two key tiles ahead, into the buffer this P leaves
          if (in_range(rg[t], j + 2)) ok = issue_s(t, j + 2);
        }
      }
      // TMEM must be quiescent before it is released
      mma_commit(&s.drain);
      mbar_wait_drain(&s.drain, 0, p.wait_limit);
    }
  } else if (warp < 8) {
    // ===================================================== softmax warpgroups
    const int t = warp >> 2;       // query tile of this warpgroup
    const int quarter = warp & 3;  // TMEM lanes [32 quarter, 32 quarter + 32)
    const int r = quarter * 32 + lane;
    const int mt = m0 + t * BM;
    const int i = mt + r;  // row inside its sequence
    const bool row_ok = i < len_q;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t col_o = tmem + lane_off + 256 + t * DV;
    const TileRange my = t ? rg[1] : rg[0];
    // rows past the end read the last row (their output is dropped)
    const float* brow = p.bias + bidx * p.bias_bstride + ((long long)h * p.Nq + min(i, len_q - 1)) * p.Nk;
    const float sc2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int step = 0; step < my.n; ++step) {
      const int b = step & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s.s_full[t][b], (step >> 1) & 1, ab));
      if (!ok) break;
      tc_fence_after();
      const uint32_t col_s = tmem + lane_off + t * 128 + b * 64;
      const int kbase = (my.jb + step) * KT;
      // tile on an edge of the visible band, or ragged: keys outside [lo, hi) are hidden
      const bool edge =
          (kbase + KT > len_k) || (kbase + KT - 1 > mt + diag + p.win_r) || (kbase < mt + BM - 1 + diag - p.win_l);
      const int hi = min(len_k, i + diag + p.win_r + 1) - kbase;
      const int lo = i + diag - p.win_l - kbase;
      // every score of the row in registers: x = s * scale * log2(e) + bias * log2(e)
      uint32_t sr[KT];
      tmem_ld32(col_s, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(col_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      reg_fence(sr);
      if constexpr (BT) {
        // this row of the staged block: 16-byte chunk c of each 32-key box sits
        // at chunk c ^ (r & 7) of the row (128-byte swizzle), so the 32 rows of
        // a warp spread over all banks; then the buffer goes back to the producer
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&s.bias_full[t], step & 1, ab)))) break;
        const uint32_t brow_s = smem_u32(s.bias[t]) + r * 128;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float bb[4];
            asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                         : "=f"(bb[0]), "=f"(bb[1]), "=f"(bb[2]), "=f"(bb[3])
                         : "r"(brow_s + half * (BM * 128) + ((c ^ (r & 7)) << 4)));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int key = 32 * half + 4 * c + e;
              sr[key] = __float_as_uint(fmaf(bb[e], kLog2e, __uint_as_float(sr[key]) * sc2));
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.bias_empty[t]);
      } else {
        // the next key tile's bias row into L2 while this one is worked on (two
        // 128-byte lines, clamped inside the row); whole tiles of 16-byte
        // aligned rows as float4 (a lane reads its own row)
        if (step + 1 < my.n) {
#pragma unroll
          for (int u = 0; u < 2; ++u)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(brow + min(kbase + KT + 32 * u, len_k - 1)));
        }
        if (p.bias_vec4 && kbase + KT <= len_k) {  // warp-uniform
          const float4* b4 = reinterpret_cast<const float4*>(brow + kbase);
#pragma unroll
          for (int c4 = 0; c4 < KT / 4; ++c4) {
            const float4 bv = __ldg(b4 + c4);
            const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
              sr[4 * c4 + u] = __float_as_uint(fmaf(bb[u], kLog2e, __uint_as_float(sr[4 * c4 + u]) * sc2));
          }
        } else {
#pragma unroll
          for (int c = 0; c < KT; ++c)
            sr[c] = __float_as_uint(fmaf(__ldg(brow + min(kbase + c, len_k - 1)), kLog2e, __uint_as_float(sr[c]) * sc2));
        }
      }
      if (edge) {
#pragma unroll
        for (int c = 0; c < KT; ++c)
          if (c >= hi || c < lo) sr[c] = 0xff800000u;  // -inf
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int c = 0; c < KT; c += 2) {
        mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
        mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
      }
      const float mx = fmaxf(mx0, mx1);
      const bool move = mx > m + kRescaleThreshold;
      const float m_next = move ? mx : m;
      const float alpha = move ? ex2(m - m_next) : 1.f;
      const float neg_m = m_next == -INFINITY ? 0.f : -m_next;
      float rs0 = 0.f, rs1 = 0.f;
      // P over the score columns already read: 32 keys -> 16 bf16 pairs per store
#pragma unroll
      for (int c = 0; c < KT / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = __uint_as_float(sr[c * 32 + 2 * e]), x1 = __uint_as_float(sr[c * 32 + 2 * e + 1]);
          const float p0 = ex2(x0 + neg_m);
          const float p1 = ex2(x1 + neg_m);
          rs0 += p0;
          rs1 += p1;
          pk[e] = pack_bf16(p0, p1);
        }
        tmem_st16(col_s + c * 16, pk);
      }
      l = l * alpha + (rs0 + rs1);
      m = m_next;
      // O may be rescaled once the previous key tile's P V is complete: the
      // scores of the next key tile were issued after it, and at the last key
      // tile pv_last is committed after it
      if (step > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        const bool done = step + 1 < my.n ? mbar_wait(&s.s_full[t][(step + 1) & 1], ((step + 1) >> 1) & 1, ab)
                                          : mbar_wait(&s.pv_last[t], 0, ab);
        if (!(ok = __all_sync(0xffffffffu, done))) break;
        tc_fence_after();
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
      if (lane == 0) mbar_arrive(&s.p_full[t][b]);
    }
    // ---- epilogue: O / l -> bf16, LSE (natural log)
    if (ok && my.n > 0) ok = __all_sync(0xffffffffu, mbar_wait(&s.o_done[t], 0, ab));
    tc_fence_after();
    if (ok) {
      // a row with no visible key (m never left -inf) is empty
      const bool empty = !(l > 0.f) || m == -INFINITY;
      const float inv_l = empty ? 0.f : 1.f / l;
      __nv_bfloat16* orow = p.o + bidx * p.o_bstride + ((long long)(q_off + i) * p.Hq + h) * DV;
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
      if (row_ok)
        p.lse[bidx * p.lse_bstride + (long long)h * p.lse_hstride + q_off + i] =
            empty ? -INFINITY : (m + __log2f(l)) * kLn2;
    }
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

template <int D, bool BT>
int launch_db_t(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                const CUtensorMap& mb, const FwdParams& p, cudaStream_t st) {
  const size_t smem = sizeof(DBSmem<D, BT>) + 1024;
  static_assert(sizeof(DBSmem<D, BT>) + 1024 <= 232448, "shared memory");
  auto kern = fwd_db_kernel<D, BT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const unsigned nblk = (g.Nq + 2 * BM - 1) / (2 * BM);
  const dim3 grid = p.batch_inner ? dim3(g.B, nblk, g.Hq) : dim3(nblk, g.Hq, g.B);
  if (grid.y > 65535 || grid.z > 65535) return ATTN_ERR_UNSUPPORTED;
  record_kernel_event(ATTN_KERNEL_FWD, 0, st);
  kern<<<grid, kThreadsOf<BT>, smem, st>>>(mq, mk, mv, mb, p);
  record_kernel_event(ATTN_KERNEL_FWD, 1, st);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_fwd_db(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const FwdParams& p, cudaStream_t st) {
  const int dv = g.Dv ? g.Dv : g.D;
  if (!g.bias || g.alibi || g.cu_q || p.num_splits != 1 || dv != g.D) return ATTN_ERR_UNSUPPORTED;
  // bias rows staged by TMA when they can be: 16-byte aligned base, rows and
  // batch stride (the same test as the vector loads); a 4-D view (key, query
  // row, head, batch), one batch when the batch shares the bias
  // (a view the tensor map cannot describe falls back to the direct loads)
  CUtensorMap mb;
  std::memset(&mb, 0, sizeof(mb));
  bool bt = p.bias_vec4;
  if (bt) {
    const uint64_t hs = (uint64_t)g.Nq * g.Nk;
    const uint64_t dims[4] = {(uint64_t)g.Nk, (uint64_t)g.Nq, (uint64_t)g.Hq, g.bias_bstride ? (uint64_t)g.B : 1};
    const uint64_t str[3] = {(uint64_t)g.Nk * 4, hs * 4, (g.bias_bstride ? (uint64_t)g.bias_bstride : g.Hq * hs) * 4};
    const uint32_t box[4] = {32, BM, 1, 1};
    bt = encode_tmap(&mb, g.bias, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dims, str, box) == ATTN_OK;
  }
  if (g.D == 128) return bt ? launch_db_t<128, true>(g, mq, mk, mv, mb, p, st)
                            : launch_db_t<128, false>(g, mq, mk, mv, mb, p, st);
  if (g.D == 64) return bt ? launch_db_t<64, true>(g, mq, mk, mv, mb, p, st)
                           : launch_db_t<64, false>(g, mq, mk, mv, mb, p, st);
  return ATTN_ERR_UNSUPPORTED;
}

}  // namespace attn
