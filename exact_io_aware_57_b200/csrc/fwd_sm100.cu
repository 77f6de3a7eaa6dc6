// Forward attention on sm_100a tensor cores.
//
// One CTA owns a tile of 128 query rows of one (batch or sequence, head) and
// streams 128-key tiles of K and V past it ("Attention IO tiling" lesson card,
// The mechanism: Q/K/V are cut into on-chip-sized tiles; each score tile
// updates the per-row softmax state and the rescaled value sum, then is
// dropped rather than stored).
//
//   warp 0      TMA producer: Q once, then K_j / V_j into a 3- or 4-stage smem ring
//   warp 1      TMEM owner + single-thread tcgen05.mma issuer
//   warps 2..5  softmax warpgroup: thread t owns query row t (TMEM lane t)
//
// TMEM (512 columns x 128 lanes x 32 bit):
//   [  0,128) S buffer 0   [128,256) S buffer 1     (fp32 scores, S = Q K_j^T)
//   [256,256+D) O accumulator (fp32)
//   [384,448) P buffer 0   [448,512) P buffer 1     (bf16 pairs, A operand of P V_j)
//
// Per key tile j the softmax thread of row i forms t = s * scale * log2(e)
// (+ bias * log2(e)), a reference max m' (moved to max_j t only when that
// exceeds m by more than 2^8), p = 2^(t - m'), l' = 2^(m - m') l + sum p
// ("Softmax does not need the matrix", "Carry the Normalizer", in base 2),
// writes P to TMEM and -- once the previous P V has landed -- rescales the O
// accumulator by 2^(m - m') when the reference moved.  V and O may have their
// own width DV (d_v).  The
// MMA warp then accumulates O += P V_j.  O / l and LSE = (m + log2 l) ln 2 are
// written once, after the last tile (the division by l happens a single time,
// as in the same page's lab).
// Causal and local (sliding-window) attention: only the KV tiles that hold a
// key visible from some row of the tile are loaded ("Understanding
// FlashAttention Pt 1", contents 3.5 tile skipping and 4.2 local attention);
// the mask is applied only on tiles that straddle the visible band.
// Split-KV: with num_splits > 1 the grid's z index also runs over splits of
// the keys (split_len keys each, a multiple of the tile); every CTA then
// writes its exact partial result -- O_t normalised in fp32 and LSE_t -- and a
// separate merge combines the splits with weights exp(LSE_t - LSE), the
// rescale-and-add of "Softmax does not need the matrix", "Carry the
// Normalizer", applied to whole splits.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace attn {

namespace {

constexpr int BM = 128;          // query rows per CTA
constexpr int BN = 128;          // keys per KV tile
// K/V shared-memory stages: as many as fit beside the Q tile in 227 KB (at
// most four).  DV is the width of V and O (d_v), D that of Q and K.
template <int D, int DV>
constexpr int kStages = (D == 128 && DV == 128) ? 3 : 4;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
constexpr float kRescaleThreshold = 8.f;  // log2 units: P stays <= 256

template <int D, int DV>
struct FwdSmem {
  static constexpr int NST = kStages<D, DV>;
  static constexpr int kTileBytes = BM * D * 2;    // 128 rows x D bf16 (Q, K)
  static constexpr int kVTileBytes = BN * DV * 2;  // 128 rows x DV bf16 (V)
  alignas(1024) uint8_t q[kTileBytes];
  alignas(1024) uint8_t k[NST][kTileBytes];
  alignas(1024) uint8_t v[NST][kVTileBytes];
  uint64_t q_full;
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, drain;
  uint32_t tmem_base;
  int abort_flag;
};



// Keep the compiler from using TMEM-loaded registers before tcgen05.wait::ld.
template <int N>
ATTN_DEVINL void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

template <int D, int DV, int BIAS, bool FAST, bool PARTIAL>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Smem = FwdSmem<D, DV>;
  constexpr int NST = Smem::NST;
  constexpr int KB = D / 64;  // 64-column (128-byte) blocks per row
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

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
  // keys [kv_begin, kv_end) hold every key visible from rows m0 .. m0 + BM - 1
  // ... clipped to this CTA's split of the keys
  const int kv_end = min(PARTIAL ? min(len_k, (split + 1) * p.split_len) : len_k, m0 + BM + diag + p.win_r);
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
      mbar_init(&s.p_full[i], 4);
    }
    mbar_init(&s.pv_done, 1);
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
      mbar_expect_tx(&s.q_full, Smem::kTileBytes);
#pragma unroll
      for (int kb = 0; kb < KB; ++kb)
        tma_load_4d(s.q + kb * BM * 128, &tm_q, &s.q_full, kb * 64, h, q_off + m0, bidx);
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % NST;
        const uint32_t ph = (j / NST) & 1;
        if (!mbar_wait(&s.k_empty[st], ph ^ 1, ab)) break;
        mbar_expect_tx(&s.k_full[st], Smem::kTileBytes);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
          tma_load_4d(s.k[st] + kb * BN * 128, &tm_k, &s.k_full[st], kb * 64, hk, k_off + (j_first + j) * BN, bidx);
        ++issued_k;
        if (!mbar_wait(&s.v_empty[st], ph ^ 1, ab)) break;
        mbar_expect_tx(&s.v_full[st], Smem::kVTileBytes);
#pragma unroll
        for (int kb = 0; kb < DV / 64; ++kb)
          tma_load_4d(s.v[st] + kb * BN * 128, &tm_v, &s.v_full[st], kb * 64, hk, k_off + (j_first + j) * BN, bidx);
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
      constexpr uint32_t idesc_s = idesc_bf16(BM, BN, 0, 0);   // Q: K-major, K_j: K-major
      constexpr uint32_t idesc_pv = idesc_bf16(BM, DV, 0, 1);  // P: TMEM, V_j: MN-major
      const uint32_t q_addr = smem_u32(s.q);
      auto issue_s = [&](int j) -> bool {
        const int buf = j & 1, st = j % NST;
        if (!mbar_wait(&s.k_full[st], (j / NST) & 1, ab)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(s.k[st]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          mma_ss(tmem + kColS + buf * BN, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024),
                 idesc_s, kk > 0);
        }
        mma_commit(&s.s_full[buf]);
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
        const int st2 = (j + 2) % NST;
        if (next && !mbar_wait(&s.k_full[st2], ((j + 2) / NST) & 1, ab)) break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(s.v[st]), k_addr = smem_u32(s.k[st2]);
        // O += P_j V_j interleaved with S_{j+2} = Q K_{j+2}^T: two independent
        // accumulators keep the tensor pipe busy (a chain of MMAs into one
        // accumulator waits on each previous result)
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ts(tmem + kColO, tmem + kColP + buf * 64 + kk * 8, sdesc_sw128(v_addr + kk * 2048, BN * 128, 1024),
                 idesc_pv, (j > 0 || kk > 0));
          if (next && kk < D / 16) {
            const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
            mma_ss(tmem + kColS + buf * BN, sdesc_sw128(q_addr + off, 16, 1024),
                   sdesc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0);
          }
        }
        mma_commit(&s.pv_done);
        mma_commit(&s.v_empty[st]);
        if (next) {
          mma_commit(&s.s_full[buf]);
          mma_commit(&s.k_empty[st2]);
        }
      }
      // TMEM must be quiescent before it is released
      mma_commit(&s.drain);
      mbar_wait_drain(&s.drain, 0, p.wait_limit);
    }
  } else {
    // ===================================================== softmax warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int i = m0 + r;                 // row inside its sequence
    const bool row_ok = i < len_q;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float* brow = nullptr;  // rows past the end read the last row (their output is dropped)
    if constexpr (BIAS == kBiasDense)
      brow = p.bias + bidx * p.bias_bstride + ((long long)h * p.Nq + min(i, len_q - 1)) * p.Nk;
    float neg_slope2 = 0.f;  // ALiBi: B = -slope |key - (i + diag)|, in log2 units
    if constexpr (BIAS == kBiasAlibi) neg_slope2 = -__ldg(p.alibi + h) * kLog2e;
    // m: the reference max of the row (log2 units) that P and l are expressed
    // against.  It only moves when a tile's max exceeds it by more than
    // kRescaleThreshold, so P <= 2^threshold and O is rescaled rarely; the
    // final O / l and LSE do not depend on which reference was used.
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int buf = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s.s_full[buf], (j >> 1) & 1, ab));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[BN];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + kColS + buf * BN + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      reg_fence(sr);
      const int kbase = (j_first + j) * BN;
      if constexpr (!FAST) {
        // general scores: t = s * scale * log2(e) (+ bias * log2(e))
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          float x = __uint_as_float(sr[c]) * p.scale_log2;
          if constexpr (BIAS == kBiasDense) x = fmaf(__ldg(brow + min(kbase + c, len_k - 1)), kLog2e, x);
          if constexpr (BIAS == kBiasAlibi) x = fmaf(neg_slope2, fabsf(static_cast<float>(kbase + c - i - diag)), x);
          sr[c] = __float_as_uint(x);
        }
      }
      if ((kbase + BN > len_k) || (kbase + BN - 1 > m0 + diag + p.win_r) ||
          (kbase < m0 + BM - 1 + diag - p.win_l)) {
        // tile on an edge of the visible band, or ragged: hide invisible keys
        const int hi = min(len_k, i + diag + p.win_r + 1) - kbase;
        const int lo = i + diag - p.win_l - kbase;
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
      if constexpr (FAST) mx *= p.scale_log2;  // scale > 0: max commutes with it
      const bool move = mx > m + kRescaleThreshold;
      const float m_next = move ? mx : m;
      const float alpha = move ? ex2(m - m_next) : 1.f;
      const float neg_m = m_next == -INFINITY ? 0.f : -m_next;
      float rs0 = 0.f, rs1 = 0.f;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN / 2; ++c) {
        float p0, p1;
        if constexpr (FAST) {
          p0 = ex2(fmaf(__uint_as_float(sr[2 * c]), p.scale_log2, neg_m));
          p1 = ex2(fmaf(__uint_as_float(sr[2 * c + 1]), p.scale_log2, neg_m));
        } else {
          p0 = ex2(__uint_as_float(sr[2 * c]) + neg_m);
          p1 = ex2(__uint_as_float(sr[2 * c + 1]) + neg_m);
        }
        rs0 += p0;
        rs1 += p1;
        pk[c] = pack_bf16(p0, p1);
      }
      l = l * alpha + (rs0 + rs1);
      m = m_next;
      if (j > 0) {
        // P V_{j-1} must be done before O is rescaled and before the P buffer
        // it read two steps ago is reused.
        ok = __all_sync(0xffffffffu, mbar_wait(&s.pv_done, (j - 1) & 1, ab));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < DV / 32; ++c) {
            uint32_t orr[32];
            tmem_ld32(tmem + lane_off + kColO + c * 32, orr);
            tmem_wait_ld();
            reg_fence(orr);
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
            tmem_st32(tmem + lane_off + kColO + c * 32, orr);
          }
        }
      }
      tmem_st32(tmem + lane_off + kColP + buf * 64, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st32(tmem + lane_off + kColP + buf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.p_full[buf]);
    }
    // ---- epilogue: O / l -> bf16, LSE (natural log)
    if (ok && n_kv > 0) ok = __all_sync(0xffffffffu, mbar_wait(&s.pv_done, (n_kv - 1) & 1, ab));
    tc_fence_after();
    if (ok) {
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.o + bidx * p.o_bstride + ((long long)(q_off + i) * p.Hq + h) * DV;
      float* prow = nullptr;
      if constexpr (PARTIAL) prow = p.o_part + split * p.part_o_stride + bidx * p.o_bstride +
                                    ((long long)(q_off + i) * p.Hq + h) * DV;
#pragma unroll
      for (int c = 0; c < DV / 32; ++c) {
        uint32_t orr[32];
        if (n_kv > 0) {
          tmem_ld32(tmem + lane_off + kColO + c * 32, orr);
          tmem_wait_ld();
          reg_fence(orr);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = 0u;
        }
        if constexpr (PARTIAL) {  // split partial: fp32
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
        const float lse = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
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

template <int D, int DV, int BIAS, bool FAST, bool PARTIAL = false>
int launch_fwd_t(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                 const FwdParams& p, cudaStream_t st) {
  // At least half of the SM's shared memory, so that a second CTA never waits
  // on the 512 TMEM columns this one holds.
  const size_t smem = std::max<size_t>(sizeof(FwdSmem<D, DV>) + 1024, 116 * 1024);
  auto kern = fwd_sm100_kernel<D, DV, BIAS, FAST, PARTIAL>;
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

}  // namespace

int launch_fwd_sm100(const TcGeom& g, __nv_bfloat16* o, float* lse, cudaStream_t st, const SplitKV* split) {
  // 4-D views (d, head, row, batch); packed inputs are one batch of `total` rows.
  const int B = g.cu_q ? 1 : g.B;
  const int dv = g.Dv ? g.Dv : g.D;  // width of V and O
  CUtensorMap mq, mk, mv;
  const uint32_t box[4] = {64, 1, 128, 1};
  {
    const uint64_t dims[4] = {(uint64_t)g.D, (uint64_t)g.Hq, (uint64_t)g.Nq, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)g.D * 2, (uint64_t)g.Hq * g.D * 2, (uint64_t)g.Nq * g.Hq * g.D * 2};
    if (encode_tmap_bf16(&mq, g.q, 4, dims, str, box) != ATTN_OK) return ATTN_ERR_CUDA;
  }
  {
    const uint64_t dims[4] = {(uint64_t)g.D, (uint64_t)g.Hkv, (uint64_t)g.Nk, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)g.D * 2, (uint64_t)g.Hkv * g.D * 2, (uint64_t)g.Nk * g.Hkv * g.D * 2};
    if (encode_tmap_bf16(&mk, g.k, 4, dims, str, box) != ATTN_OK) return ATTN_ERR_CUDA;
    const uint64_t dv_dims[4] = {(uint64_t)dv, (uint64_t)g.Hkv, (uint64_t)g.Nk, (uint64_t)B};
    const uint64_t dv_str[3] = {(uint64_t)dv * 2, (uint64_t)g.Hkv * dv * 2, (uint64_t)g.Nk * g.Hkv * dv * 2};
    if (encode_tmap_bf16(&mv, g.v, 4, dv_dims, dv_str, box) != ATTN_OK) return ATTN_ERR_CUDA;
  }
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.bias = g.bias;
  p.bias_bstride = g.bias_bstride;
  p.alibi = g.alibi;
  p.cu_q = g.cu_q;
  p.cu_k = g.cu_k;
  p.max_nq = g.max_nq;
  p.max_nk = g.max_nk;
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.Nq = g.Nq;
  p.Nk = g.Nk;
  p.o_bstride = g.cu_q ? 0 : (long long)g.Nq * g.Hq * dv;
  p.lse_bstride = g.cu_q ? 0 : (long long)g.Hq * g.Nq;
  p.lse_hstride = g.Nq;  // packed: Nq is the total row count
  p.scale_log2 = g.scale * kLog2e;
  p.causal = g.causal;
  p.win_l = win_left(g.window_left);
  p.win_r = win_right(g.causal, g.window_right);
  p.num_splits = 1;
  p.split_len = g.Nk;
  if (split) {  // dense inputs only
    p.num_splits = split->num_splits;
    p.split_len = split->split_len;
    p.o_part = split->o_part;
    p.lse_part = split->lse_part;
    p.part_o_stride = (long long)g.B * g.Nq * g.Hq * g.D;
    p.part_lse_stride = (long long)g.B * g.Hq * g.Nq;
  }
  p.status = device_status_ptr();
  p.wait_limit = kWaitLimitCycles;
  if (!p.status) return ATTN_ERR_CUDA;
  // FAST: no bias and a positive scale, so the row max can be taken on raw scores
  const bool fast = !g.bias && !g.alibi && g.scale > 0.f;
#ifndef ATTN_FWD_SINGLE_TILE
  if (dv != g.D && (split || g.bias || g.alibi)) return ATTN_ERR_UNSUPPORTED;
  return launch_fwd_pp(g, mq, mk, mv, p, g.bias ? kBiasDense : g.alibi ? kBiasAlibi : kBiasNone, fast,
                       split != nullptr, st);
#else
  if (dv != g.D) {  // value width of its own: dense or packed, no bias, one pass
    if (split || g.bias || g.alibi) return ATTN_ERR_UNSUPPORTED;
    if (g.D == 128)
      return fast ? launch_fwd_t<128, 64, kBiasNone, true>(g, mq, mk, mv, p, st)
                  : launch_fwd_t<128, 64, kBiasNone, false>(g, mq, mk, mv, p, st);
    return fast ? launch_fwd_t<64, 128, kBiasNone, true>(g, mq, mk, mv, p, st)
                : launch_fwd_t<64, 128, kBiasNone, false>(g, mq, mk, mv, p, st);
  }
  if (split) {  // no bias on this path
    if (g.D == 64)
      return fast ? launch_fwd_t<64, 64, kBiasNone, true, true>(g, mq, mk, mv, p, st)
                  : launch_fwd_t<64, 64, kBiasNone, false, true>(g, mq, mk, mv, p, st);
    return fast ? launch_fwd_t<128, 128, kBiasNone, true, true>(g, mq, mk, mv, p, st)
                : launch_fwd_t<128, 128, kBiasNone, false, true>(g, mq, mk, mv, p, st);
  }
  if (g.D == 64) {
    if (g.bias) return launch_fwd_t<64, 64, kBiasDense, false>(g, mq, mk, mv, p, st);
    if (g.alibi) return launch_fwd_t<64, 64, kBiasAlibi, false>(g, mq, mk, mv, p, st);
    return fast ? launch_fwd_t<64, 64, kBiasNone, true>(g, mq, mk, mv, p, st)
                : launch_fwd_t<64, 64, kBiasNone, false>(g, mq, mk, mv, p, st);
  }
  if (g.bias) return launch_fwd_t<128, 128, kBiasDense, false>(g, mq, mk, mv, p, st);
  if (g.alibi) return launch_fwd_t<128, 128, kBiasAlibi, false>(g, mq, mk, mv, p, st);
  return fast ? launch_fwd_t<128, 128, kBiasNone, true>(g, mq, mk, mv, p, st)
              : launch_fwd_t<128, 128, kBiasNone, false>(g, mq, mk, mv, p, st);
#endif
}

}  // namespace attn
