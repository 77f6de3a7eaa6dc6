// Backward attention on sm_100a tensor cores: P is rebuilt tile by tile from
// the per-row log-sum-exp kept by the forward instead of being stored ("Attention
// IO tiling" lesson card, The mechanism, last step; "Understanding FlashAttention
// Pt 1", section 3.6 in its contents).  The pages print no gradient formulas; the
// kernel forms the exact gradient of softmax(scale QK^T + B)V:
//   P = exp(scale S + B - LSE),  dV = P^T dO,  dP = dO V^T,
//   dS = P o (dP - D) with D_i = dO_i . O_i,  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three launches:
//   bwd_pre    D_i = dO_i . O_i (fp32) and zero the fp32 dQ accumulator
//   bwd_main   one CTA per (128-key tile, KV head, batch or packed sequence);
//              K_j and V_j stay in shared memory, dK_j and dV_j accumulate in
//              TMEM over every query tile and every query head of the group
//   bwd_dq     dQ = scale * accumulator -> bf16
//
// bwd_main roles (10 warps):
//   warp 0      TMA producer (K_j, V_j once; Q_i, dO_i per step) + LSE/D rows,
//               and the TMA reduce-add of each staged dQ tile
//   warp 1      TMEM owner + single-thread tcgen05.mma issuer
//   warps 2..9  two groups of four; TMEM lane t is key row t for P^T / dS^T and
//               the dK/dV epilogue, and query row t for the dQ tile.  Group g
//               takes queries [64g, 64g+64) of P^T / dS^T and columns
//               [gD/2, (g+1)D/2) of dQ, dK and dV, so every SM sub-partition
//               runs two warps of each elementwise phase.
// D is the width of Q, K, dQ, dK and DV that of V, O, dO, dV (equal except
// for attn_bwd_dv).  TMEM columns: [0,128) S^T (then P^T as bf16 pairs in
// [0,64)), [128,256) dP^T (then the dQ tile), [256,256+DV) dV,
// [256+DV,256+DV+D) dK.
// Per step (query head h, query tile i):
//   MMA   dP^T = V_j dO_i^T once the previous dQ has left TMEM (S^T of this step
//         was issued earlier, see below)
//   WGs   P^T = 2^(scale log2e S^T + log2e B^T - log2e LSE) -> TMEM (bf16,
//         each group over its own half of the S^T columns), overlapping the
//         dP^T MMAs; P^T also stays in registers for dS^T;
//         dS^T = P^T o (dP^T - D) -> shared memory (bf16, 128B-swizzled)
//   MMA   dV += P^T dO_i (P^T from TMEM) once P^T is there, overlapping dS^T;
//         S^T of the next step = K_j Q_{i+1}^T as soon as Q_{i+1} has arrived
//         (the scores columns are free once P^T has been read out), so the
//         elementwise groups find the next scores ready; then dQ_i = dS K_j
//         and, after it, dK += dS^T Q_i
//   WGs   dQ_i -> the step's own Q_i/dO_i buffers as soon as the dQ MMAs are
//         done (the Q_i half only after dK has read Q_i); the next dP^T may
//         start in its columns while dK runs.  The producer adds the staged
//         tile into the fp32 accumulator with TMA bulk reductions and refills
//         the buffers only after those have read them, so the reduction
//         overlaps the next step instead of holding it up.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace attn {

namespace {

constexpr int BM = 128;   // query rows per step
constexpr int BN = 128;   // keys per CTA
constexpr int NSTQ = 2;   // Q/dO stages
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColST = 0, kColDPT = 128, kColDV = 256;
// One exponential of P^T in kBwdEmuEvery goes to the FMA pipe (ex2_poly) on
// tiles without a mask (measured: 1 in 8 helps a little, 1 in 4 hurts).
#ifndef ATTN_BWD_EX2_EMU_EVERY
#define ATTN_BWD_EX2_EMU_EVERY 8
#endif
constexpr int kBwdEmuEvery = ATTN_BWD_EX2_EMU_EVERY;

// D: width of Q, K, dQ, dK; DV: width of V, O, dO, dV.  The fp32 dQ tile of a
// step (D / 32 boxes of 128 rows x 32 columns, 16 KB each) is staged in that
// step's Q and dO buffers (D / 64 + DV / 64 boxes) and, when D > DV, in an
// extra buffer for the boxes they cannot hold.
template <int D, int DV>
struct BwdSmem {
  static constexpr int kKBytes = 128 * D * 2;
  static constexpr int kVBytes = 128 * DV * 2;
  static constexpr int kQBoxes = D / 64, kDoBoxes = DV / 64;
  static constexpr int kXBoxes = D / 32 > kQBoxes + kDoBoxes ? D / 32 - kQBoxes - kDoBoxes : 0;
  alignas(1024) uint8_t k[kKBytes];
  alignas(1024) uint8_t v[kVBytes];
  alignas(1024) uint8_t q[NSTQ][kKBytes];
  alignas(1024) uint8_t dout[NSTQ][kVBytes];
  alignas(1024) uint8_t ds[128 * 128 * 2];  // dS^T, [key][query] in two 64-column blocks
  alignas(1024) uint8_t dqx[NSTQ][kXBoxes > 0 ? kXBoxes * 128 * 128 : 16];
  alignas(16) float nlse2[NSTQ][BM];        // -log2(e) * LSE of the step's query rows (-inf: no key)
  alignas(16) float drow[NSTQ][BM];         // D_i of the step's query rows
  uint64_t kv_full, q_full[NSTQ], do_full[NSTQ], staged[NSTQ];
  uint64_t st_full, dp_full, pt_ready, ds_ready, dq_done, dkq_done, tmem_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct BwdParams {
  const float* lse;
  const float* drow;
  float* dq_acc;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* bias;
  long long bias_bstride;
  int batch_inner;  // grid (batch, key tile, KV head): the batch elements sharing one bias run together
  const float* alibi;
  const int* cu_q;  // packed sequences: prefix offsets (device), or null
  const int* cu_k;
  int max_nq, max_nk;  // packed: bounds on the sequence lengths
  int n_z;             // batch elements or packed sequences
  int Hq, Hkv, Nq, Nk;
  float scale, scale_log2;
  int causal;
  int win_l, win_r;  // key j visible from query i iff i + diag - win_l <= j <= i + diag + win_r
  int* status;
  long long wait_limit;
};

template <int N>
ATTN_DEVINL void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}


// out[tile] += smem tile (fp32), completion tracked by bulk groups
ATTN_DEVINL void tma_reduce_add_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
ATTN_DEVINL void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
ATTN_DEVINL void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
ATTN_DEVINL void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
ATTN_DEVINL void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

ATTN_DEVINL void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Phase A -- P^T for one key row (this thread) and 128 queries, 32 at a time:
//   P^T = 2^(scale log2e s + log2e B - log2e LSE), written back into TMEM as
// bf16 pairs over the S^T columns already read (A operand of dV += P^T dO).
// MASK zeroes queries this key is hidden from (query i sees key kj iff
// kj - lo_off <= i <= kj + hi_off, i.e. i + diag - win_l <= kj <= i + diag + win_r;
// padding rows and keys).
// bb: the dense bias of these 32 queries for this key (loaded ahead by the caller).
template <bool MASK, int BIAS>
ATTN_DEVINL void p_chunk(int c, const uint32_t (&sr)[32], uint32_t st_col, const float* nlse2, float scale_log2,
                         const float (&bb)[32], float neg_slope2, int i0, int len_q, int kj, int len_k,
                         int lo_off, int hi_off, int bias_diag, uint32_t (&pk)[16]) {
  const float4* nl4 = reinterpret_cast<const float4*>(nlse2 + c * 32);
  const int q0 = i0 + c * 32;
  int vis_lo = 0, vis_hi = 32;  // queries q0 + e, vis_lo <= e < vis_hi, see this key
  if constexpr (MASK) {
    vis_lo = kj - lo_off - q0;
    vis_hi = min(min(32, len_q - q0), kj + hi_off - q0 + 1);
    if (kj >= len_k) vis_hi = 0;
  }
#pragma unroll
  for (int e4 = 0; e4 < 8; ++e4) {
    const float4 nl = nl4[e4];
    const float nlv[4] = {nl.x, nl.y, nl.z, nl.w};
    float pv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e4 * 4 + u;
      float t = fmaf(__uint_as_float(sr[e]), scale_log2, nlv[u]);
      if constexpr (BIAS == kBiasDense) t = fmaf(bb[e], kLog2e, t);
      if constexpr (BIAS == kBiasAlibi) t = fmaf(neg_slope2, fabsf(static_cast<float>(kj - q0 - e - bias_diag)), t);
      // unmasked tiles (every t finite): one exponential in kBwdEmuEvery on the FMA pipe
      float pe = (!MASK && kBwdEmuEvery > 0 && e % kBwdEmuEvery == kBwdEmuEvery - 1) ? ex2_poly(t) : ex2(t);
      if constexpr (MASK) pe = (e >= vis_lo && e < vis_hi) ? pe : 0.f;
      pv[u] = pe;
    }
    pk[2 * e4] = pack_bf16(pv[0], pv[1]);
    pk[2 * e4 + 1] = pack_bf16(pv[2], pv[3]);
  }
  // chunk c (32 queries, 16 columns of bf16 pairs) over S^T columns this thread
  // has already read: [16c, 16c+16) for group 0's chunks 0, 1 and [16c+32,
  // 16c+48) for group 1's chunks 2, 3, so neither group writes over the
  // other's scores
  tmem_st16(st_col + c * 16 + (c & 2) * 16, pk);
}

// Group g's half of phase A: queries [64g, 64g+64), chunks 2g and 2g+1, read
// from S^T columns [64g, 64g+64) and written back as P^T into the first half of
// the same columns (p_chunk), so the two groups need not wait for each other.
// keep: this thread's P^T as bf16 pairs (chunk 2g in [0,16), chunk 2g+1 in [16,32)).
template <bool MASK, int BIAS>
ATTN_DEVINL void bwd_p_half(int grp, uint32_t st_col, const float* nlse2, float scale_log2, const float (&bb)[64],
                            float neg_slope2, int i0, int len_q, int kj, int len_k, int lo_off, int hi_off,
                            int bias_diag, uint32_t (&keep)[32]) {
  const int c0 = 2 * grp;
  uint32_t ra[32], rb[32];
  tmem_ld32(st_col + c0 * 32, ra);
  tmem_ld32(st_col + (c0 + 1) * 32, rb);
  tmem_wait_ld();
  reg_fence(ra);
  reg_fence(rb);
  p_chunk<MASK, BIAS>(c0, ra, st_col, nlse2, scale_log2, *reinterpret_cast<const float(*)[32]>(&bb[0]), neg_slope2,
                      i0, len_q, kj, len_k, lo_off, hi_off, bias_diag, *reinterpret_cast<uint32_t(*)[16]>(&keep[0]));
  p_chunk<MASK, BIAS>(c0 + 1, rb, st_col, nlse2, scale_log2, *reinterpret_cast<const float(*)[32]>(&bb[32]),
                      neg_slope2, i0, len_q, kj, len_k, lo_off, hi_off, bias_diag,
                      *reinterpret_cast<uint32_t(*)[16]>(&keep[16]));
}

// Phase B -- dS^T = P^T (dP^T - D) from the bf16 P^T and dP^T, into the
// 128B-swizzled shared tile (K-major for dK += dS^T Q, MN-major for dQ = dS K).
ATTN_DEVINL void ds_chunk(int c, const uint32_t (&pr)[16], const uint32_t (&dpr)[32], const float* drow,
                          uint32_t ds_row, int r) {
  const float4* dr4 = reinterpret_cast<const float4*>(drow + c * 32);
  uint32_t dk[16];
#pragma unroll
  for (int e4 = 0; e4 < 8; ++e4) {
    const float4 dr = dr4[e4];
    const float drv[4] = {dr.x, dr.y, dr.z, dr.w};
    float dsv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e4 * 4 + u;
      const uint32_t pair = pr[e >> 1];
      const float pe = __uint_as_float((e & 1) ? (pair & 0xffff0000u) : (pair << 16));
      dsv[u] = pe * (__uint_as_float(dpr[e]) - drv[u]);
    }
    dk[2 * e4] = pack_bf16(dsv[0], dsv[1]);
    dk[2 * e4 + 1] = pack_bf16(dsv[2], dsv[3]);
  }
  // 32 queries = 4 chunks of 16 bytes in 64-column block c/2
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int chunk = (c & 1) * 4 + u;  // 16-byte chunk within the 128-byte row
    const uint32_t addr = ds_row + (c >> 1) * (128 * 128) + ((chunk ^ (r & 7)) << 4);
    st_shared_v4(addr, dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
  }
}

// Group g's half of phase B (chunks 2g and 2g+1): dP^T from TMEM, P^T from the
// values this thread kept in registers in phase A (`keep`), so the S^T
// columns may already hold the next step's scores.
ATTN_DEVINL void bwd_ds_half_kept(int grp, const uint32_t (&keep)[32], uint32_t dp_col, const float* drow,
                                  uint32_t ds_row, int r) {
  const int c0 = 2 * grp;
  uint32_t da[32], db[32];
  tmem_ld32(dp_col + c0 * 32, da);
  tmem_ld32(dp_col + (c0 + 1) * 32, db);
  tmem_wait_ld();
  reg_fence(da);
  reg_fence(db);
  ds_chunk(c0, *reinterpret_cast<const uint32_t(*)[16]>(&keep[0]), da, drow, ds_row, r);
  ds_chunk(c0 + 1, *reinterpret_cast<const uint32_t(*)[16]>(&keep[16]), db, drow, ds_row, r);
}

template <int D, int DV, int BIAS>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using Smem = BwdSmem<D, DV>;
  constexpr int KB = D / 64, KBV = DV / 64;
  constexpr uint32_t kColDK = kColDV + DV;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // grid (key tile, KV head, batch or sequence): the key tiles of groups of four
  // (batch, head) pairs are interleaved (grouped_unit), so that the heavy causal
  // tiles start early while the CTAs running at one time still share a few
  // heads' Q / dO tiles in L2 (a heaviest-first order across all heads measured
  // 13 % slower on the causal workload).  When the batch elements share a
  // dense bias (grid (batch, key tile, KV head)), a group is every batch
  // element of two KV heads, so the ones reading the same bias run side by side.
  int n_tile, hk, zz;
  if (p.batch_inner) {
    const int nb = (int)gridDim.x;
    int u;
    grouped_unit((int)gridDim.y, nb * p.Hkv, 2 * nb, n_tile, u);
    hk = u / nb, zz = u % nb;
  } else {
    int u;
    grouped_unit((int)gridDim.x, (int)(gridDim.y * gridDim.z), 4, n_tile, u);
    hk = u % p.Hkv, zz = u / p.Hkv;
  }
  const int n0 = n_tile * BN;
  // dense: batch element b; packed: sequence zz at rows q_off / k_off of batch 0
  int b = zz, q_off = 0, k_off = 0, len_q = p.Nq, len_k = p.Nk;
  if (p.cu_q) {
    // invalid offsets: reported in the status word, nothing read or written
    if (!packed_seq(p.cu_q, zz, p.Nq, p.max_nq, p.status, q_off, len_q) ||
        !packed_seq(p.cu_k, zz, p.Nk, p.max_nk, p.status, k_off, len_k))
      return;
    b = 0;
  }
  if (n0 >= len_k) return;  // past this sequence's keys: uniform, before any barrier or TMEM use
  const int diag = len_k - len_q;  // query i is aligned with key i + diag
  const int G = p.Hq / p.Hkv;
  // query rows that see at least one key of n0 .. n0 + BN - 1
  const int first_row = max(0, n0 - diag - p.win_r);
  const int last_row = min(len_q - 1, n0 + BN - 1 - diag + p.win_l);
  const int i_first = first_row / BM;
  const int per_head = last_row >= first_row ? last_row / BM - i_first + 1 : 0;
  const int n_steps = G * per_head;

  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the swizzle needs 1024-byte aligned tiles
    if (threadIdx.x == 0) atomicExch(p.status, ATTN_ERR_CUDA);
    return;
  }
  if (threadIdx.x == 0) {
    s.abort_flag = 0;
    mbar_init(&s.kv_full, 1);
    for (int i = 0; i < NSTQ; ++i) {
      mbar_init(&s.q_full[i], 1 + 32);   // TMA transaction arrive + 32 producer lanes (LSE rows)
      mbar_init(&s.do_full[i], 1 + 32);  // TMA transaction arrive + 32 producer lanes (D rows)
      mbar_init(&s.staged[i], 8);   // the eight elementwise warps, dQ tile staged
    }
    mbar_init(&s.st_full, 1);
    mbar_init(&s.dp_full, 1);
    mbar_init(&s.ds_ready, 8);
    mbar_init(&s.pt_ready, 8);
    mbar_init(&s.dq_done, 1);
    mbar_init(&s.dkq_done, 1);
    mbar_init(&s.tmem_free, 8);
    mbar_init(&s.drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const Abort ab{&s.abort_flag, p.status, p.wait_limit};

  // staging place of fp32 dQ box c (columns 32c .. 32c + 31) of stage st
  auto dq_box = [&](int st, int c) -> uint8_t* {
    if (c < Smem::kQBoxes) return s.q[st] + c * (128 * 128);
    if (c < Smem::kQBoxes + Smem::kDoBoxes) return s.dout[st] + (c - Smem::kQBoxes) * (128 * 128);
    return s.dqx[st] + (c - Smem::kQBoxes - Smem::kDoBoxes) * (128 * 128);
  };
  if (warp == 0) {
    // ===================================================== producer
    // Stage st of step s held the dQ tile of step s - NSTQ: before reloading
    // it, add that tile into the accumulator.  The boxes staged in the Q buffer
    // go first, as a bulk group of their own, so that Q_s (all the next scores
    // need) loads as soon as the reduction has read them; dO_s loads, on a
    // barrier of its own, once the rest has been read.
    int issued = 0;
    auto reduce_step = [&](int t) -> bool {
      const int st = t % NSTQ;
      if (!__all_sync(0xffffffffu, mbar_wait(&s.staged[st], (t / NSTQ) & 1, ab))) return false;
      if (lane == 0) {
        const int h = hk * G + t / per_head;
        const int i0 = (i_first + t % per_head) * BM;
#pragma unroll
        for (int c = 0; c < Smem::kQBoxes; ++c)
          tma_reduce_add_4d(&tm_dq, dq_box(st, c), c * 32, h, q_off + i0, b);
        bulk_commit();
#pragma unroll
        for (int c = Smem::kQBoxes; c < D / 32; ++c)
          tma_reduce_add_4d(&tm_dq, dq_box(st, c), c * 32, h, q_off + i0, b);
        bulk_commit();
      }
      __syncwarp();
      return true;
    };
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_dq);
      if (n_steps > 0) {
        mbar_expect_tx(&s.kv_full, Smem::kKBytes + Smem::kVBytes);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) tma_load_4d(s.k + kb * BN * 128, &tm_k, &s.kv_full, kb * 64, hk, k_off + n0, b);
#pragma unroll
        for (int kb = 0; kb < KBV; ++kb) tma_load_4d(s.v + kb * BN * 128, &tm_v, &s.kv_full, kb * 64, hk, k_off + n0, b);
      }
    }
    bool ok = true;
    for (int step = 0; step < n_steps; ++step) {
      const int st = step % NSTQ;
      const int h = hk * G + step / per_head;
      const int i0 = (i_first + step % per_head) * BM;
      // LSE / D rows of this step into registers first (their latency overlaps
      // the wait for the stage)
      const long long row0 = ((long long)b * p.Hq + h) * p.Nq + q_off;
      float l2v[BM / 32], drv[BM / 32];
#pragma unroll
      for (int e = 0; e < BM / 32; ++e) {
        const int qi = i0 + lane + 32 * e;
        l2v[e] = -INFINITY;
        drv[e] = 0.f;
        if (qi < len_q) {
          const float lse = p.lse[row0 + qi];
          l2v[e] = lse == -INFINITY ? -INFINITY : -lse * kLog2e;
          drv[e] = p.drow[row0 + qi];
        }
      }
      if (step >= NSTQ && !(ok = reduce_step(step - NSTQ))) break;
      if (lane == 0) {
        if (step >= NSTQ) bulk_wait_read1();  // the Q buffer's boxes have been read
        mbar_expect_tx(&s.q_full[st], Smem::kKBytes);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
          tma_load_4d(s.q[st] + kb * BM * 128, &tm_q, &s.q_full[st], kb * 64, h, q_off + i0, b);
      }
#pragma unroll
      for (int e = 0; e < BM / 32; ++e) s.nlse2[st][lane + 32 * e] = l2v[e];
      mbar_arrive(&s.q_full[st]);
      if (lane == 0) {
        if (step >= NSTQ) bulk_wait_read0();  // and the rest
        mbar_expect_tx(&s.do_full[st], Smem::kVBytes);
#pragma unroll
        for (int kb = 0; kb < KBV; ++kb)
          tma_load_4d(s.dout[st] + kb * BM * 128, &tm_do, &s.do_full[st], kb * 64, h, q_off + i0, b);
      }
#pragma unroll
      for (int e = 0; e < BM / 32; ++e) s.drow[st][lane + 32 * e] = drv[e];
      mbar_arrive(&s.do_full[st]);
      ++issued;
    }
    // the last NSTQ dQ tiles
    for (int t = max(0, n_steps - NSTQ); ok && t < n_steps; ++t) ok = reduce_step(t);
    if (lane == 0) {
      bulk_wait0();  // every reduction has completed before the CTA exits
      if (s.abort_flag) {
        if (n_steps > 0) mbar_wait_drain(&s.kv_full, 0, p.wait_limit);
        for (int j = max(0, issued - NSTQ); j < issued; ++j) {
          mbar_wait_drain(&s.q_full[j % NSTQ], (j / NSTQ) & 1, p.wait_limit);
          mbar_wait_drain(&s.do_full[j % NSTQ], (j / NSTQ) & 1, p.wait_limit);
        }
      }
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    if (lane == 0 && n_steps > 0) {
      constexpr uint32_t idesc_s = idesc_bf16(BN, BM, 0, 0);    // K_j / V_j (K-major) x Q_i / dO_i (K-major)
      constexpr uint32_t idesc_dv = idesc_bf16(BN, DV, 0, 1);   // P^T (K-major) x dO_i (MN-major)
      constexpr uint32_t idesc_kv = idesc_bf16(BN, D, 0, 1);    // dS^T (K-major) x Q_i (MN-major)
      constexpr uint32_t idesc_dq = idesc_bf16(BM, D, 1, 1);    // dS (MN-major) x K_j (MN-major)
      const uint32_t k_addr = smem_u32(s.k), v_addr = smem_u32(s.v), ds_addr = smem_u32(s.ds);
      // S^T(t) = K_j Q_t^T into [0, 128) (over P^T of the step before, whose dV
      // MMA was issued earlier by this thread: tcgen05.mma executes in issue order)
      auto s_mmas = [&](uint32_t q_addr) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          mma_ss(tmem + kColST, sdesc_sw128(k_addr + off, 16, 1024), sdesc_sw128(q_addr + off, 16, 1024), idesc_s,
                 kk > 0);
        }
      };
      // The next step's scores: S^T(t + 1) over P^T(t) once dV(t) (issued before,
      // executed in issue order) has read it; the elementwise groups keep P^T in
      // registers for dS^T, so the S^T columns are free after the P^T phase.
      int s_issued = 0;
      auto next_s = [&](int t, bool block) -> bool {  // issue S^T(t) if its Q has arrived (or wait for it)
        if (t >= n_steps || s_issued != t) return true;
        const int st1 = t % NSTQ;
        const uint32_t par = (t / NSTQ) & 1;
        if (block) {
          if (!mbar_wait(&s.q_full[st1], par, ab)) return false;
        } else if (!mbar_try_wait(&s.q_full[st1], par)) {
          return true;
        }
        tc_fence_after();
        s_mmas(smem_u32(s.q[st1]));
        // its completion also implies that the MMAs issued before it are done
        mma_commit(&s.st_full);
        ++s_issued;
        return true;
      };
      bool ok = mbar_wait(&s.kv_full, 0, ab);
      if (ok) ok = next_s(0, true);
      for (int step = 0; ok && step < n_steps; ++step) {
        const int st = step % NSTQ;
        const uint32_t q_addr = smem_u32(s.q[st]), do_addr = smem_u32(s.dout[st]);
        // dP^T = V_j dO_i^T where dQ of the previous step was, once that has left
        if (step > 0 && !(ok = mbar_wait(&s.tmem_free, (step - 1) & 1, ab))) break;
        if (!(ok = mbar_wait(&s.do_full[st], (step / NSTQ) & 1, ab))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          mma_ss(tmem + kColDPT, sdesc_sw128(v_addr + off, 16, 1024), sdesc_sw128(do_addr + off, 16, 1024), idesc_s,
                 kk > 0);
        }
        mma_commit(&s.dp_full);
        // dV += P^T dO_i as soon as P^T is in TMEM; it overlaps the dS^T phase
        if (!(ok = mbar_wait(&s.pt_ready, step & 1, ab))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)  // queries [16kk, 16kk+16): columns kk*8 (+32 for group 1's half)
          mma_ts(tmem + kColDV, tmem + kColST + kk * 8 + (kk >= 4 ? 32 : 0),
                 sdesc_sw128(do_addr + kk * 2048, BM * 128, 1024), idesc_dv, (step > 0 || kk > 0));
        if (!(ok = next_s(step + 1, false))) break;
        // dQ_i = dS K_j (the dS^T tile read MN-major), then dK += dS^T Q_i, once
        // dS^T is in shared memory
        if (!(ok = mbar_wait(&s.ds_ready, step & 1, ab))) break;
        if (!(ok = next_s(step + 1, false))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ss(tmem + kColDPT, sdesc_sw128(ds_addr + kk * 2048, 128 * 128, 1024),
                 sdesc_sw128(k_addr + kk * 2048, BN * 128, 1024), idesc_dq, kk > 0);
        // dQ_i may leave TMEM, and dO_i (last read by dV) is free
        mma_commit(&s.dq_done);
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          mma_ss(tmem + kColDK, sdesc_sw128(ds_addr + off, 16, 1024), sdesc_sw128(q_addr + kk * 2048, BM * 128, 1024),
                 idesc_kv, (step > 0 || kk > 0));
        }
        // every MMA of the step is done: Q_i is free, and the dS^T tile may be
        // rewritten
        mma_commit(&s.dkq_done);
        if (!(ok = next_s(step + 1, true))) break;
      }
      mma_commit(&s.drain);
      mbar_wait_drain(&s.drain, 0, p.wait_limit);
    }
  } else {
    // ===================================================== elementwise groups
    const int grp = (warp - 2) >> 2;  // 0: warps 2..5, 1: warps 6..9
    const int quarter = warp & 3;     // TMEM lanes [32 quarter, 32 quarter + 32)
    const int r = quarter * 32 + lane;
    const int kj = n0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t ds_row = smem_u32(s.ds) + r * 128;
    bool ok = true;
    uint32_t keep[32];  // this thread's P^T of the step (bf16 pairs), reused by the dS^T phase
    // dQ_t (this thread: query row r, columns [grp D/2, grp D/2 + D/2)) from TMEM
    // into step t's own Q_t / dO_t buffers (box c: columns 32c .. 32c+31, 16 KB,
    // 128B-swizzled like the TMA map) for the producer's reduce-add
    // Group 0's boxes are exactly the Q_t buffer, which dK (issued after dQ)
    // still reads: that group waits for dK before it stores; group 1's boxes
    // (the dO_t buffer, and the extra buffer when D > DV) are free once dQ is.
    // The next dS^T tile is written only after the next dP^T, whose commit
    // follows this step's dK.
    auto drain = [&](int t) -> bool {
      const int st = t % NSTQ;
      if (!__all_sync(0xffffffffu, mbar_wait(&s.dq_done, t & 1, ab))) return false;
      tc_fence_after();
      uint32_t a[D / 2];
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tmem_ld32(tmem + lane_off + kColDPT + grp * (D / 2) + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&a[c * 32]));
      tmem_wait_ld();
      reg_fence(a);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.tmem_free);
      if (grp == 0 && !__all_sync(0xffffffffu, mbar_wait(&s.dkq_done, t & 1, ab))) return false;
#pragma unroll
      for (int cl = 0; cl < D / 64; ++cl) {
        const int c = grp * (D / 64) + cl;
        const uint32_t row = smem_u32(dq_box(st, c)) + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = cl * 32 + 4 * u;
          st_shared_v4(row + ((u ^ (r & 7)) << 4), a[e], a[e + 1], a[e + 2], a[e + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.staged[st]);
      return true;
    };
    // the dense bias of this key and the group's 64 queries of step t, loaded a
    // step ahead (before the previous step's dQ staging) so that its latency
    // passes there (rows past the end read the last row; their P^T is masked)
    float bb[64];
    auto load_bias = [&](int t) {
      if constexpr (BIAS == kBiasDense) {
        const int ht = hk * G + t / per_head, qg = (i_first + t % per_head) * BM + 64 * grp;
        const float* bcol = p.bias + b * p.bias_bstride + (long long)ht * p.Nq * p.Nk + min(kj, len_k - 1);
#pragma unroll
        for (int e = 0; e < 64; ++e) bb[e] = __ldg(bcol + (long long)min(qg + e, len_q - 1) * p.Nk);
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) bb[e] = 0.f;
      }
    };
    if (n_steps > 0) load_bias(0);
    for (int step = 0; step < n_steps; ++step) {
      const int st = step % NSTQ;
      const int h = hk * G + step / per_head;
      const int i0 = (i_first + step % per_head) * BM;
      // S^T is in TMEM; q_full of this stage (LSE rows) completed before, and
      // do_full (D rows) before dP^T
      ok = __all_sync(0xffffffffu, mbar_wait(&s.st_full, step & 1, ab));
      if (!ok) break;
      tc_fence_after();
      // tile-level (warp-uniform) condition: the chunk routines hold
      // warp-collective tcgen05 instructions, so every lane must take the same one
      const bool need_mask = (n0 + BN > len_k) || (i0 + BM > len_q) || (n0 + BN - 1 > i0 + diag + p.win_r) ||
                             (n0 < i0 + BM - 1 + diag - p.win_l);
      float neg_slope2 = 0.f;
      if constexpr (BIAS == kBiasAlibi) neg_slope2 = -__ldg(p.alibi + h) * kLog2e;
      const uint32_t st_col = tmem + lane_off + kColST, dp_col = tmem + lane_off + kColDPT;
      if (need_mask)
        bwd_p_half<true, BIAS>(grp, st_col, s.nlse2[st], p.scale_log2, bb, neg_slope2, i0, len_q, kj, len_k,
                               diag + p.win_r, p.win_l - diag, diag, keep);
      else
        bwd_p_half<false, BIAS>(grp, st_col, s.nlse2[st], p.scale_log2, bb, neg_slope2, i0, len_q, kj, len_k, 0, 0,
                                diag, keep);
      tmem_wait_st();
      // P^T is in TMEM: the dV MMAs (and the next step's scores) may start
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.pt_ready);
      // dP^T of this step
      ok = __all_sync(0xffffffffu, mbar_wait(&s.dp_full, step & 1, ab));
      if (!ok) break;
      tc_fence_after();
      bwd_ds_half_kept(grp, keep, dp_col, s.drow[st], ds_row, r);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.ds_ready);
      if (step + 1 < n_steps) load_bias(step + 1);
      if (!(ok = drain(step))) break;
    }
    // ---- epilogue: dV (columns [grp DV/2, grp DV/2 + DV/2)) and dK (scaled,
    // columns [grp D/2, grp D/2 + D/2)) of key row r.  The MMA warp commits
    // `drain` after its last MMA
    if (ok && n_steps > 0) ok = __all_sync(0xffffffffu, mbar_wait(&s.drain, 0, ab));
    tc_fence_after();
    if (ok) {
      const long long key = ((long long)b * p.Nk + k_off + kj) * p.Hkv + hk;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int W = half == 0 ? DV : D;
        const uint32_t col0 = (half == 0 ? kColDV : kColDK) + grp * (W / 2);
        const float mul = half == 0 ? 1.f : p.scale;
        __nv_bfloat16* dst = (half == 0 ? p.dv : p.dk) + key * W + grp * (W / 2);
#pragma unroll
        for (int c = 0; c < W / 64; ++c) {
          uint32_t a[32];
          if (n_steps > 0) {
            tmem_ld32(tmem + lane_off + col0 + c * 32, a);
            tmem_wait_ld();
            reg_fence(a);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) a[e] = 0u;
          }
          uint32_t pkd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pkd[e] = pack_bf16(__uint_as_float(a[2 * e]) * mul, __uint_as_float(a[2 * e + 1]) * mul);
          if (kj < len_k) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// D_i = dO_i . O_i (fp32, rows of DV) and zeroed dQ accumulator rows (D).  One
// warp per (b, n, h) row.
template <int D, int DV>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout, float* __restrict__ drow,
                                                      float* __restrict__ dq_acc, int B, int Hq, int Nq) {
  constexpr int EV = DV / 32, EQ = D / 32;  // elements per lane (2 or 4)
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= (long long)B * Nq * Hq) return;
  float acc = 0.f;
  const __nv_bfloat16* orow = o + row * DV + lane * EV;
  const __nv_bfloat16* drw = dout + row * DV + lane * EV;
#pragma unroll
  for (int e = 0; e < EV; ++e) acc = fmaf(__bfloat162float(orow[e]), __bfloat162float(drw[e]), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  float* q = dq_acc + row * D + lane * EQ;
#pragma unroll
  for (int e = 0; e < EQ; ++e) q[e] = 0.f;
  if (lane == 0) {
    const int h = (int)(row % Hq);
    const long long bn = row / Hq;
    const int n = (int)(bn % Nq), bb = (int)(bn / Nq);
    drow[((long long)bb * Hq + h) * Nq + n] = acc;
  }
}

// dQ = scale * accumulator, fp32 -> bf16, 8 elements per thread.
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                     long long n8, float scale) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 c = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  reinterpret_cast<uint4*>(dq)[i] = make_uint4(pack_bf16(a.x * scale, a.y * scale), pack_bf16(a.z * scale, a.w * scale),
                                               pack_bf16(c.x * scale, c.y * scale), pack_bf16(c.z * scale, c.w * scale));
}

template <int D, int DV, int BIAS>
int launch_main_t(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const CUtensorMap& mdo, const CUtensorMap& mdq, const BwdParams& p, cudaStream_t st) {
  const size_t smem = std::max<size_t>(sizeof(BwdSmem<D, DV>), 116 * 1024);
  auto kern = bwd_main_kernel<D, DV, BIAS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const unsigned n_tiles = ((g.cu_q ? g.max_nk : g.Nk) + BN - 1) / BN;
  const dim3 grid = p.batch_inner ? dim3(p.n_z, n_tiles, g.Hkv) : dim3(n_tiles, g.Hkv, p.n_z);
  if (grid.y > 65535 || grid.z > 65535) return ATTN_ERR_UNSUPPORTED;
  record_kernel_event(ATTN_KERNEL_BWD, 0, st);
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, mdo, mdq, p);
  record_kernel_event(ATTN_KERNEL_BWD, 1, st);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

int launch_bwd_sm100(const TcGeom& g, const __nv_bfloat16* o, const float* lse, const __nv_bfloat16* dout,
                     __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, float* dq_acc, float* Drow,
                     cudaStream_t st) {
  // packed sequences are one batch of g.Nq / g.Nk total rows
  const int dvw = g.Dv ? g.Dv : g.D;  // width of V, O, dO, dV
  // 1) D and zeroed accumulator
  {
    const long long rows = (long long)g.B * g.Nq * g.Hq;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    if (g.D == 64 && dvw == 64)
      bwd_pre_kernel<64, 64><<<blocks, 256, 0, st>>>(o, dout, Drow, dq_acc, g.B, g.Hq, g.Nq);
    else if (g.D == 128 && dvw == 128)
      bwd_pre_kernel<128, 128><<<blocks, 256, 0, st>>>(o, dout, Drow, dq_acc, g.B, g.Hq, g.Nq);
    else if (g.D == 128)
      bwd_pre_kernel<128, 64><<<blocks, 256, 0, st>>>(o, dout, Drow, dq_acc, g.B, g.Hq, g.Nq);
    else
      bwd_pre_kernel<64, 128><<<blocks, 256, 0, st>>>(o, dout, Drow, dq_acc, g.B, g.Hq, g.Nq);
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  // 2) main
  CUtensorMap mq, mk, mv, mdo, mdq;
  const uint32_t box[4] = {64, 1, 128, 1};
  {
    const uint64_t dims[4] = {(uint64_t)g.D, (uint64_t)g.Hq, (uint64_t)g.Nq, (uint64_t)g.B};
    const uint64_t str[3] = {(uint64_t)g.D * 2, (uint64_t)g.Hq * g.D * 2, (uint64_t)g.Nq * g.Hq * g.D * 2};
    if (encode_tmap_bf16(&mq, g.q, 4, dims, str, box) != ATTN_OK) return ATTN_ERR_CUDA;
    const uint64_t dv_dims[4] = {(uint64_t)dvw, (uint64_t)g.Hq, (uint64_t)g.Nq, (uint64_t)g.B};
    const uint64_t dv_str[3] = {(uint64_t)dvw * 2, (uint64_t)g.Hq * dvw * 2, (uint64_t)g.Nq * g.Hq * dvw * 2};
    if (encode_tmap_bf16(&mdo, dout, 4, dv_dims, dv_str, box) != ATTN_OK) return ATTN_ERR_CUDA;
    // fp32 accumulator: 32 floats (128 bytes) x 128 rows per box
    const uint64_t str32[3] = {(uint64_t)g.D * 4, (uint64_t)g.Hq * g.D * 4, (uint64_t)g.Nq * g.Hq * g.D * 4};
    const uint32_t box32[4] = {32, 1, 128, 1};
    if (encode_tmap(&mdq, dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dims, str32, box32) != ATTN_OK)
      return ATTN_ERR_CUDA;
  }
  {
    const uint64_t dims[4] = {(uint64_t)g.D, (uint64_t)g.Hkv, (uint64_t)g.Nk, (uint64_t)g.B};
    const uint64_t str[3] = {(uint64_t)g.D * 2, (uint64_t)g.Hkv * g.D * 2, (uint64_t)g.Nk * g.Hkv * g.D * 2};
    if (encode_tmap_bf16(&mk, g.k, 4, dims, str, box) != ATTN_OK) return ATTN_ERR_CUDA;
    const uint64_t dv_dims[4] = {(uint64_t)dvw, (uint64_t)g.Hkv, (uint64_t)g.Nk, (uint64_t)g.B};
    const uint64_t dv_str[3] = {(uint64_t)dvw * 2, (uint64_t)g.Hkv * dvw * 2, (uint64_t)g.Nk * g.Hkv * dvw * 2};
    if (encode_tmap_bf16(&mv, g.v, 4, dv_dims, dv_str, box) != ATTN_OK) return ATTN_ERR_CUDA;
  }
  BwdParams p{};
  p.lse = lse;
  p.drow = Drow;
  p.dq_acc = dq_acc;
  p.dk = dk;
  p.dv = dv;
  p.bias = g.bias;
  p.bias_bstride = g.bias_bstride;
  // a dense bias shared by the batch elements: run them side by side so that
  // they read each bias tile from L2 instead of each from memory
  p.batch_inner = g.bias && g.bias_bstride == 0 && !g.cu_q && g.B > 1;
  p.alibi = g.alibi;
  p.cu_q = g.cu_q;
  p.cu_k = g.cu_k;
  p.max_nq = g.max_nq;
  p.max_nk = g.max_nk;
  p.n_z = g.cu_q ? g.num_seqs : g.B;
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.Nq = g.Nq;
  p.Nk = g.Nk;
  p.scale = g.scale;
  p.scale_log2 = g.scale * kLog2e;
  p.causal = g.causal;
  p.win_l = win_left(g.window_left);
  p.win_r = win_right(g.causal, g.window_right);
  p.status = device_status_ptr();
  p.wait_limit = kWaitLimitCycles;
  if (!p.status) return ATTN_ERR_CUDA;
  int rc;
  if (dvw != g.D)  // value width of its own: no bias
    rc = (g.bias || g.alibi) ? ATTN_ERR_UNSUPPORTED
         : g.D == 128        ? launch_main_t<128, 64, kBiasNone>(g, mq, mk, mv, mdo, mdq, p, st)
                             : launch_main_t<64, 128, kBiasNone>(g, mq, mk, mv, mdo, mdq, p, st);
  else if (g.D == 64)
    rc = g.bias    ? launch_main_t<64, 64, kBiasDense>(g, mq, mk, mv, mdo, mdq, p, st)
         : g.alibi ? launch_main_t<64, 64, kBiasAlibi>(g, mq, mk, mv, mdo, mdq, p, st)
                   : launch_main_t<64, 64, kBiasNone>(g, mq, mk, mv, mdo, mdq, p, st);
  else
    rc = g.bias    ? launch_main_t<128, 128, kBiasDense>(g, mq, mk, mv, mdo, mdq, p, st)
         : g.alibi ? launch_main_t<128, 128, kBiasAlibi>(g, mq, mk, mv, mdo, mdq, p, st)
                   : launch_main_t<128, 128, kBiasNone>(g, mq, mk, mv, mdo, mdq, p, st);
  if (rc) return rc;
  // 3) dQ
  const long long n8 = (long long)g.B * g.Nq * g.Hq * g.D / 8;
  bwd_dq_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(dq_acc, dq, n8, g.scale);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn
