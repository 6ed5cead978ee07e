// bwd_sm100.cu -- exact attention backward pass for B200 (sm_100a), recompute form.
//
// What it computes: the gradients of sum(O * dO) for O = softmax(scale Q K^T) V.
// The pages keep only O and the per-row statistics and rebuild the score and
// probability blocks on chip during the backward pass ("AI Bible 13", section
// 03, second axe; "FlashAttention saves IO, not N^2 work", section 3).  With the
// saved lse_i (natural log) the probabilities are P_ij = exp(scale q_i.k_j - lse_i);
// the rest is the textbook softmax vector-Jacobian product:
//     dV = P^T dO,   dP = dO V^T,   D_i = dO_i . O_i,   dS = P o (dP - D),
//     dQ = scale dS K,   dK = scale dS^T Q.
//
// Three kernels:
//   1. preprocess: D_i = dO_i . O_i (fp32) and a zeroed fp32 dQ accumulator;
//   2. main (tcgen05): one CTA per (b, h, 128-key tile); K_j and V_j stay in
//      shared memory while the CTA walks the 128-row query tiles that can see
//      them (from the causal diagonal onward).  Each query tile is processed as
//      two halves of 64 queries so that the dS warps work on one half while the
//      tensor core computes the other:
//        S^T = K Q^T and dP^T = V dO^T      (M = 128 keys, N = 64 queries)
//        P^T -> tensor memory (bf16), dS^T -> shared memory (bf16, swizzled)
//        dV += P^T dO (A from tensor memory),  dK += dS^T Q
//        dQ_tile = dS K                      (M = 128 queries, A read MN-major)
//      dQ tiles leave tensor memory through fp32 vector reductions into the
//      accumulator; dK and dV leave once, through a TMA store.
//   3. convert: dQ = bf16(scale * accumulator).
#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr int kThreads = 320;  // warp 0 TMA + stats, warp 1 MMA, warps 2-9 dS warps (two column groups)
constexpr uint32_t kTmemCols = 512;

// A query tile of 128 rows is processed in kSteps steps of kNq queries.  The
// tensor core computes step t+2's S^T and dP^T into one of two ping-pong buffers
// while the dS warps work on step t+1 and the MMAs of step t (dV, dK) run.
template <int D>
struct BwdLayout {
  static constexpr int kNq = (D == 64) ? 64 : 32;  // queries per step
  static constexpr int kSteps = 128 / kNq;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 16384;
  static constexpr int kQStages = 2;
  static constexpr int kDsBufs = (D == 64) ? 2 : 1;
  static constexpr int kDsBytes = 2 * 16384;  // [64-query atom][128 keys][64 queries] bf16, 128-byte swizzle
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;
  static constexpr int kOffDO = kOffQ + kQStages * kTileBytes;
  static constexpr int kOffDS = kOffDO + kQStages * kTileBytes;
  static constexpr int kOffStat = kOffDS + kDsBufs * kDsBytes;  // per stage: lse2[128], D[128]
  // d = 64: dQ tiles leave through an fp32 staging tile and a TMA reduce-add
  // (two 128-row x 32-column boxes, one per dS column group); d = 128 uses
  // per-thread vector reductions instead (no room for the staging tile).
  static constexpr bool kDqTma = (D == 64);
  static constexpr int kOffDQ = kOffStat + kQStages * 2 * 128 * 4;
  static constexpr int kOffBar = kOffDQ + (kDqTma ? 128 * D * 4 : 0);
  // kv_full, q_full[QS], q_empty[QS], s_full[2], p_full[2], ds_free[DSB], dq_full, dq_empty, dkv_done, epi,
  // dq_staged[2], dq_stage_free[2]
  static constexpr int kNumBars = 1 + 2 * kQStages + 4 + kDsBufs + 4 + 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64;
  // tensor memory columns
  __host__ __device__ static constexpr uint32_t tm_st(int b) { return b * kNq; }           // S^T buffers (P^T bf16 over them)
  __host__ __device__ static constexpr uint32_t tm_dpt(int b) { return 2 * kNq + b * kNq; }  // dP^T buffers
  static constexpr uint32_t kTmDV = 4 * kNq;
  static constexpr uint32_t kTmDK = 4 * kNq + D;
  static constexpr uint32_t kTmDQ = 4 * kNq + 2 * D;
  static_assert(kTmDQ + D <= kTmemCols, "tensor memory budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct BwdArgs {
  const float* lse;
  const float* delta;
  float* dq_acc;
  int* status;
  int B, H, Nq, Nk;
  int causal;
  float scale;
  float scale_log2;
  int n_kv_tiles;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void bwd_timeout(int* status, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicCAS(status, 0, kStatusTimeout);
}

__device__ __forceinline__ bool warp_wait_b(uint64_t* bar, uint32_t parity, unsigned long long timeout_ns) {
  bool ok = true;
  if (lane_id() == 0) ok = mbar_wait(bar, parity, timeout_ns);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// X^T step = A . B_step^T  (M = 128 keys, N = kNq queries, K = D), both K-major.
// Used for S^T = K Q^T and dP^T = V dO^T.
template <int D>
__device__ __forceinline__ void issue_step_scores(uint32_t d_tmem, uint32_t a_smem, uint32_t b_step_smem) {
  using L = BwdLayout<D>;
  constexpr uint32_t idesc = idesc_bf16_f32(128, L::kNq, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
    umma_ss(d_tmem, sdesc_sw128(a_smem + off, 16, 1024), sdesc_sw128(b_step_smem + off, 16, 1024), idesc,
            kk > 0 ? 1u : 0u);
  }
}

// acc (+)= A . B_step where B_step is kNq rows (queries) x D, read MN-major (N = D).
// A is P^T in tensor memory (kAFromTmem) or dS^T in shared memory, K-major.  In
// tensor memory each dS column group keeps its P^T over the start of its own S^T
// columns: queries [g*kNq/2, (g+1)*kNq/2) of the step sit at columns g*kNq/2 ..
// g*kNq/2 + kNq/4 (two bf16 per column).
template <int D, bool kAFromTmem>
__device__ __forceinline__ void issue_step_acc(uint32_t acc_tmem, uint32_t a, uint32_t b_step_smem, bool first) {
  using L = BwdLayout<D>;
  constexpr int kHalf = L::kNq / 2, kPerGroup = kHalf / 16;  // 16-query k-steps per column group
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
  for (int kk = 0; kk < L::kNq / 16; ++kk) {
    const uint64_t bdesc = sdesc_sw128(b_step_smem + kk * 2048, 16384, 1024);
    const uint32_t acc = (first && kk == 0) ? 0u : 1u;
    if (kAFromTmem)
      umma_ts(acc_tmem, a + (kk / kPerGroup) * kHalf + (kk % kPerGroup) * 8, bdesc, idesc, acc);
    else
      umma_ss(acc_tmem, sdesc_sw128(a + kk * 32, 16, 1024), bdesc, idesc, acc);
  }
}

// dQ tile = dS . K  (M = 128 queries, N = D, K = 128 keys); dS and K both MN-major.
template <int D>
__device__ __forceinline__ void issue_dq(uint32_t dq_tmem, uint32_t ds_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, true, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    umma_ss(dq_tmem, sdesc_sw128(ds_smem + kk * 2048, 16384, 1024), sdesc_sw128(k_smem + kk * 2048, 16384, 1024),
            idesc, kk > 0 ? 1u : 0u);
  }
}

// P and dS for one key row and kN consecutive queries:
//   p = exp2(s * scale_log2 - lse2_q),  ds = p * (dp - D_q)
// packed to bf16 pairs.  `stat` holds -lse2 (128 floats) then -D (128 floats) of
// the query tile, already offset to the first query.  With kMask, queries before
// `qrel_min` (relative to the first query) and all queries of an out-of-range key
// get p = 0.
template <int kN, bool kMask>
__device__ __forceinline__ void ds_block(const uint32_t (&sv)[kN], const uint32_t (&dp)[kN], uint32_t stat,
                                         float scale_log2, bool key_ok, int qrel_min, uint32_t (&pk)[kN / 2],
                                         uint32_t (&dsk)[kN / 2]) {
  const float2 sc2 = make_float2(scale_log2, scale_log2);
#pragma unroll
  for (int c = 0; c < kN; c += 4) {
    const float4 nl = ld_shared_f4(stat + c * 4);
    const float4 nd = ld_shared_f4(stat + 512 + c * 4);
    const float2 x0 = ffma2(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sc2,
                            make_float2(nl.x, nl.y));
    const float2 x1 = ffma2(make_float2(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])), sc2,
                            make_float2(nl.z, nl.w));
    float2 p0 = make_float2(ex2(x0.x), ex2(x0.y));
    float2 p1 = make_float2(ex2(x1.x), ex2(x1.y));
    if (kMask) {
      if (!key_ok || c + 0 < qrel_min) p0.x = 0.f;
      if (!key_ok || c + 1 < qrel_min) p0.y = 0.f;
      if (!key_ok || c + 2 < qrel_min) p1.x = 0.f;
      if (!key_ok || c + 3 < qrel_min) p1.y = 0.f;
    }
    const float2 t0 = fadd2(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), make_float2(nd.x, nd.y));
    const float2 t1 = fadd2(make_float2(__uint_as_float(dp[c + 2]), __uint_as_float(dp[c + 3])),
                            make_float2(nd.z, nd.w));
    const float2 d0 = fmul2(p0, t0), d1 = fmul2(p1, t1);
    pk[c / 2] = pack_bf16x2(p0.x, p0.y);
    pk[c / 2 + 1] = pack_bf16x2(p1.x, p1.y);
    dsk[c / 2] = pack_bf16x2(d0.x, d0.y);
    dsk[c / 2 + 1] = pack_bf16x2(d1.x, d1.y);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                    const __grid_constant__ CUtensorMap tmDQacc, const BwdArgs a) {
  using L = BwdLayout<D>;
  constexpr int kNq = L::kNq, kSteps = L::kSteps, kHalf = kNq / 2;  // kHalf: queries per dS warp per step
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* bar_kv_full = bars;
  uint64_t* bar_q_full = bars + 1;
  uint64_t* bar_q_empty = bar_q_full + L::kQStages;
  uint64_t* bar_s_full = bar_q_empty + L::kQStages;
  uint64_t* bar_p_full = bar_s_full + 2;
  uint64_t* bar_ds_free = bar_p_full + 2;
  uint64_t* bar_dq_full = bar_ds_free + L::kDsBufs;
  uint64_t* bar_dq_empty = bar_dq_full + 1;
  uint64_t* bar_dkv_done = bar_dq_empty + 1;
  uint64_t* bar_epi = bar_dkv_done + 1;
  uint64_t* bar_dq_staged = bar_epi + 1;
  uint64_t* bar_dq_stage_free = bar_dq_staged + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 8);

  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t sbase = smem_u32(smem);

  // work: key tile j of head (b, h); heavy (early) key tiles first under the causal mask
  const int bh_count = a.B * a.H;
  const int j = blockIdx.x / bh_count;
  const int bh = blockIdx.x - j * bh_count;
  const int b = bh / a.H, h = bh - (bh / a.H) * a.H;
  const int n_qtiles = (a.Nq + 127) >> 7;
  int i_first = 0;
  if (a.causal) i_first = max(0, j * 128 - (a.Nk - a.Nq)) >> 7;
  const int n_iters = n_qtiles - i_first;
  const int n_steps = n_iters * kSteps;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv_full, 1);
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar_q_full + s, 2);  // TMA bytes + the producer's stats
      mbar_init(bar_q_empty + s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full + t, 1);
      mbar_init(bar_p_full + t, 8);  // one arrival per dS warp
    }
    for (int s = 0; s < L::kDsBufs; ++s) mbar_init(bar_ds_free + s, 1);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_empty, 8);
    mbar_init(bar_dkv_done, 1);
    mbar_init(bar_epi, 8);
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar_dq_staged + g, 4);
      mbar_init(bar_dq_stage_free + g, 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const size_t stat_row = ((size_t)b * a.H + h) * a.Nq;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer: TMA tiles + lse/D
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_kv_full, 2 * L::kTileBytes);
      for (int bx = 0; bx < L::kBoxes; ++bx) {
        tma_load_4d(smem + L::kOffK + bx * L::kBoxBytes, &tmK, bar_kv_full, bx * 64, h, j * 128, b);
        tma_load_4d(smem + L::kOffV + bx * L::kBoxBytes, &tmV, bar_kv_full, bx * 64, h, j * 128, b);
      }
    }
    for (int it = 0; it < n_iters; ++it) {
      const int st = it % L::kQStages;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(bar_q_empty + st, ((it / L::kQStages) & 1) ^ 1, a.timeout_ns) && !*abort_flag;
      if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) {
        if (lane == 0) bwd_timeout(a.status, abort_flag);
        break;
      }
      const int q0 = (i_first + it) * 128;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar_q_full + st, 2 * L::kTileBytes);
        for (int bx = 0; bx < L::kBoxes; ++bx) {
          tma_load_4d(smem + L::kOffQ + st * L::kTileBytes + bx * L::kBoxBytes, &tmQ, bar_q_full + st, bx * 64, h,
                      q0, b);
          tma_load_4d(smem + L::kOffDO + st * L::kTileBytes + bx * L::kBoxBytes, &tmDO, bar_q_full + st, bx * 64,
                      h, q0, b);
        }
      }
      // -lse in log2 units (-inf for rows past Nq or with no visible key: P = 0 there)
      // and -D, negated so that the dS warps use them as addends
      float* stat = reinterpret_cast<float*>(smem + L::kOffStat) + st * 256;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = lane + 32 * e, q = q0 + c;
        float nl2 = -INFINITY, nd = 0.f;
        if (q < a.Nq) {
          const float lse = a.lse[stat_row + q];
          nl2 = (lse == -INFINITY) ? -INFINITY : -lse * 1.4426950408889634f;
          nd = -a.delta[stat_row + q];
        }
        stat[c] = nl2;
        stat[128 + c] = nd;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_q_full + st);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar_kv_full, 0, a.timeout_ns);
      const uint32_t k_s = sbase + L::kOffK, v_s = sbase + L::kOffV;
      auto q_stage = [&](int it) { return sbase + L::kOffQ + (it % L::kQStages) * L::kTileBytes; };
      auto do_stage = [&](int it) { return sbase + L::kOffDO + (it % L::kQStages) * L::kTileBytes; };
      // S^T and dP^T of global step t into ping-pong buffer t % 2
      auto issue_scores = [&](int t) -> bool {
        const int it = t / kSteps, s = t - (t / kSteps) * kSteps;
        if (s == 0) {
          if (!mbar_wait(bar_q_full + (it % L::kQStages), (it / L::kQStages) & 1, a.timeout_ns) || *abort_flag)
            return false;
          tc_fence_after();
        }
        const int buf = t & 1;
        issue_step_scores<D>(tmem + L::tm_st(buf), k_s, q_stage(it) + s * kNq * 128);
        issue_step_scores<D>(tmem + L::tm_dpt(buf), v_s, do_stage(it) + s * kNq * 128);
        umma_commit(bar_s_full + buf);
        return true;
      };
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2 && t < n_steps && ok; ++t) ok = issue_scores(t);
      }
      for (int t = 0; t < n_steps && ok; ++t) {
        const int it = t / kSteps, s = t - (t / kSteps) * kSteps, buf = t & 1;
        if (!mbar_wait(bar_p_full + buf, (t >> 1) & 1, a.timeout_ns) || *abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ds_s = sbase + L::kOffDS + (it % L::kDsBufs) * L::kDsBytes;
        // dS^T of this step: atom (s * kNq) / 64, byte offset ((s * kNq) % 64) * 2 inside the 128-byte rows
        const uint32_t ds_step = ds_s + ((s * kNq) >> 6) * 16384 + ((s * kNq) & 63) * 2;
        issue_step_acc<D, true>(tmem + L::kTmDV, tmem + L::tm_st(buf), do_stage(it) + s * kNq * 128, t == 0);
        issue_step_acc<D, false>(tmem + L::kTmDK, ds_step, q_stage(it) + s * kNq * 128, t == 0);
        if (s == kSteps - 1) {
          if (it > 0) {  // the previous dQ tile must have left tensor memory
            if (!mbar_wait(bar_dq_empty, (it - 1) & 1, a.timeout_ns) || *abort_flag) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          issue_dq<D>(tmem + L::kTmDQ, ds_s, k_s);
          umma_commit(bar_dq_full);
          umma_commit(bar_ds_free + (it % L::kDsBufs));
          umma_commit(bar_q_empty + (it % L::kQStages));
        }
        if (t + 2 < n_steps) ok = issue_scores(t + 2);
      }
      if (!ok) bwd_timeout(a.status, abort_flag);
      umma_commit(bar_dkv_done);
    }
  } else {
    // ------------------------------------------------------------------ dS warps (thread = key)
    const uint32_t quarter = warp & 3;
    const int grp = (warp - 2) >> 2;  // column group: queries [grp * kHalf, +kHalf) of each step
    const int r = quarter * 32 + lane;
    const int key = j * 128 + r;
    const uint32_t lane_field = (quarter * 32) << 16;
    const bool key_ok = key < a.Nk;
    // first query that sees this key (a sentinel far below any query when not causal;
    // qmin - qs below must not overflow)
    const int qmin = a.causal ? key - (a.Nk - a.Nq) : -(1 << 30);
    bool ok = true;

    // dQ tile of query tile `it`: this group's D/2 columns leave tensor memory and
    // are added into the fp32 accumulator
    int drains = 0;
    auto drain_dq = [&](int it) -> bool {
      if constexpr (L::kDqTma) {
        // the staging box of this group must have been read by the previous reduce
        if (!warp_wait_b(bar_dq_stage_free + grp, (drains & 1) ^ 1, a.timeout_ns)) return false;
      }
      if (!warp_wait_b(bar_dq_full, it & 1, a.timeout_ns) || *abort_flag) return false;
      tc_fence_after();
      uint32_t g[D / 64][32];
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) tmem_ld32(tmem + lane_field + L::kTmDQ + grp * (D / 2) + cc * 32, g[cc]);
      tmem_ld_wait(g[0]);
#pragma unroll
      for (int cc = 1; cc < D / 64; ++cc) reg_pin(g[cc]);
      tc_fence_before();
      mbar_arrive_warp(bar_dq_empty);
      const int q0 = (i_first + it) * 128;
      if constexpr (L::kDqTma) {
        // row r of box grp, 128-byte swizzle; one elected thread adds the box into global memory
        const uint32_t box = sbase + L::kOffDQ + grp * 16384 + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(box + ((c ^ (r & 7)) << 4), g[0][4 * c], g[0][4 * c + 1], g[0][4 * c + 2], g[0][4 * c + 3]);
        fence_proxy_async_smem();
        mbar_arrive_warp(bar_dq_staged + grp);
        bool staged = true;
        if (quarter == 2 && lane == 0) {  // first warp of the group
          staged = mbar_wait(bar_dq_staged + grp, drains & 1, a.timeout_ns);
          if (staged) {
            tma_reduce_add_4d(&tmDQacc, smem + L::kOffDQ + grp * 16384, grp * 32, h, q0, b);
            bulk_commit_group();
            bulk_wait_group_read0();
            mbar_arrive(bar_dq_stage_free + grp);
          }
        }
        if (__shfl_sync(0xffffffffu, staged ? 1 : 0, 0) == 0) return false;
      } else {
        const int q = q0 + r;
        if (q < a.Nq) {
          float* dst = a.dq_acc + (((size_t)b * a.Nq + q) * a.H + h) * D + grp * (D / 2);
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc)
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              red_add_v4(dst + cc * 32 + e, __uint_as_float(g[cc][e]), __uint_as_float(g[cc][e + 1]),
                         __uint_as_float(g[cc][e + 2]), __uint_as_float(g[cc][e + 3]));
        }
      }
      ++drains;
      return true;
    };

    for (int t = 0; t < n_steps && ok; ++t) {
      const int it = t / kSteps, s = t - (t / kSteps) * kSteps, buf = t & 1;
      const int st = it % L::kQStages;
      const int q0 = (i_first + it) * 128;
      if (s == 0) {
        // stats of this query tile are staged with it; its dS buffer must be free
        if (!warp_wait_b(bar_q_full + st, (it / L::kQStages) & 1, a.timeout_ns) ||
            !warp_wait_b(bar_ds_free + (it % L::kDsBufs), ((it / L::kDsBufs) & 1) ^ 1, a.timeout_ns) ||
            *abort_flag) {
          ok = false;
          break;
        }
      }
      if (!warp_wait_b(bar_s_full + buf, (t >> 1) & 1, a.timeout_ns) || *abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int qs = q0 + s * kNq + grp * kHalf;  // first query of this warp's columns
      const uint32_t stat_u32 = sbase + L::kOffStat + st * 1024 + (s * kNq + grp * kHalf) * 4;
      uint32_t sv[kHalf], dp[kHalf];
      if constexpr (kHalf == 32) {
        tmem_ld32(tmem + lane_field + L::tm_st(buf) + grp * kHalf, sv);
        tmem_ld32(tmem + lane_field + L::tm_dpt(buf) + grp * kHalf, dp);
        tmem_ld_wait(sv);
        reg_pin(dp);
      } else {
        tmem_ld16(tmem + lane_field + L::tm_st(buf) + grp * kHalf, sv);
        tmem_ld16(tmem + lane_field + L::tm_dpt(buf) + grp * kHalf, dp);
        tmem_ld_wait16(sv);
        reg_pin16(dp);
      }
      const bool tile_mask = (j * 128 + 128 > a.Nk) || (a.causal && (j * 128 + 127 - (a.Nk - a.Nq) > qs));
      uint32_t pk[kHalf / 2], dk2[kHalf / 2];
      if (tile_mask)
        ds_block<kHalf, true>(sv, dp, stat_u32, a.scale_log2, key_ok, qmin - qs, pk, dk2);
      else
        ds_block<kHalf, false>(sv, dp, stat_u32, a.scale_log2, key_ok, qmin - qs, pk, dk2);
      // P^T (bf16 pairs) over the start of this group's own S^T columns (the other
      // group may still be reading its columns)
      if constexpr (kHalf == 32)
        tmem_st16(tmem + lane_field + L::tm_st(buf) + grp * kHalf, pk);
      else
        tmem_st8(tmem + lane_field + L::tm_st(buf) + grp * kHalf, pk);
      // dS^T row of this key for these queries: kHalf/8 chunks of 16 bytes, 128-byte swizzle
      const uint32_t ds_u32 = sbase + L::kOffDS + (it % L::kDsBufs) * L::kDsBytes;
      const int qt = s * kNq + grp * kHalf;  // query offset within the tile
      const uint32_t row_base = ds_u32 + (qt >> 6) * 16384 + r * 128;
#pragma unroll
      for (int c8 = 0; c8 < kHalf / 8; ++c8) {
        const int chunk = ((qt & 63) >> 3) + c8;
        st_shared_v4(row_base + ((chunk ^ (r & 7)) << 4), dk2[c8 * 4 + 0], dk2[c8 * 4 + 1], dk2[c8 * 4 + 2],
                     dk2[c8 * 4 + 3]);
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar_p_full + buf);
      // the previous query tile's dQ is complete by now (it ran before this step's scores)
      if (s == kSteps - 1 && it > 0) {
        if (!drain_dq(it - 1)) {
          ok = false;
          break;
        }
      }
    }
    if (ok && n_iters > 0) ok = drain_dq(n_iters - 1);
    if (quarter == 2 && lane == 0) bulk_wait_group0();  // reduce-adds of this thread have landed
    // ---------------------------------------------------------------- dK / dV epilogue
    // group 0 stores dK (times scale) through the K tile's smem, group 1 dV through V's
    if (ok && warp_wait_b(bar_dkv_done, 0, a.timeout_ns) && !*abort_flag) {
      tc_fence_after();
      const uint32_t src = tmem + lane_field + (grp == 0 ? L::kTmDK : L::kTmDV);
      const uint32_t dst = sbase + (grp == 0 ? L::kOffK : L::kOffV);
      const float mul = grp == 0 ? a.scale : 1.f;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(src + cc * 32, o);
        tmem_ld_wait(o);
        const int box = cc >> 1;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = (cc & 1) * 4 + q4;
          const uint32_t addr = dst + box * L::kBoxBytes + r * 128 + ((chunk ^ (r & 7)) << 4);
          const float* f = reinterpret_cast<const float*>(o) + q4 * 8;
          st_shared_v4(addr, pack_bf16x2(f[0] * mul, f[1] * mul), pack_bf16x2(f[2] * mul, f[3] * mul),
                       pack_bf16x2(f[4] * mul, f[5] * mul), pack_bf16x2(f[6] * mul, f[7] * mul));
        }
      }
      fence_proxy_async_smem();
      mbar_arrive_warp(bar_epi);
      if (warp == 2 && lane == 0) {
        if (mbar_wait(bar_epi, 0, a.timeout_ns)) {
          for (int bx = 0; bx < L::kBoxes; ++bx) {
            tma_store_4d(&tmDK, smem + L::kOffK + bx * L::kBoxBytes, bx * 64, h, j * 128, b);
            tma_store_4d(&tmDV, smem + L::kOffV + bx * L::kBoxBytes, bx * 64, h, j * 128, b);
          }
          bulk_commit_group();
          bulk_wait_group0();
        } else {
          bwd_timeout(a.status, abort_flag);
        }
      }
      __syncwarp();
    } else if (lane == 0) {
      bwd_timeout(a.status, abort_flag);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// D_i = dO_i . O_i  ([B, H, Nq] fp32) and a zeroed dQ accumulator ([B, Nq, H, D] fp32).
// One row (b, i, h) per D/8 threads, 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o,
                                                             const __nv_bfloat16* __restrict__ dout,
                                                             float* __restrict__ delta, float* __restrict__ dq_acc,
                                                             int B, int H, int Nq) {
  constexpr int kTpr = D / 8;  // threads per row
  const long long rows = (long long)B * Nq * H;
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / kTpr;
  const int part = threadIdx.x % kTpr;
  float acc = 0.f;
  if (row < rows) {
    const uint4 x = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
    const uint4 y = *reinterpret_cast<const uint4*>(dout + row * D + part * 8);
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(xs[e] << 16), __uint_as_float(ys[e] << 16), acc);
      acc = fmaf(__uint_as_float(xs[e] & 0xFFFF0000u), __uint_as_float(ys[e] & 0xFFFF0000u), acc);
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + row * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && part == 0) {
    const long long h = row % H;
    const long long bi = row / H;  // b * Nq + i
    const long long bb = bi / Nq, i = bi % Nq;
    delta[(bb * H + h) * Nq + i] = acc;
  }
}

// dq = bf16(scale * dq_acc), 8 elements per thread.
__global__ void __launch_bounds__(256) bwd_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                          long long n8, float scale) {
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n8; t += (long long)gridDim.x * blockDim.x) {
    const float4 x = reinterpret_cast<const float4*>(acc)[2 * t];
    const float4 y = reinterpret_cast<const float4*>(acc)[2 * t + 1];
    uint4 w;
    w.x = pack_bf16x2(x.x * scale, x.y * scale);
    w.y = pack_bf16x2(x.z * scale, x.w * scale);
    w.z = pack_bf16x2(y.x * scale, y.y * scale);
    w.w = pack_bf16x2(y.z * scale, y.w * scale);
    reinterpret_cast<uint4*>(dq)[t] = w;
  }
}

}  // namespace

template <int D>
static fa_status launch_bwd_impl(const BwdLaunch& L0, cudaStream_t stream) {
  using L = BwdLayout<D>;
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(bwd_main_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes) !=
        cudaSuccess)
      return FA_ERR_CUDA;
    attr_done[dev] = true;
  }
  // 1. D rows and a zeroed dQ accumulator
  {
    const long long rows = (long long)L0.B * L0.Nq * L0.H;
    const long long threads = rows * (D / 8);
    const int grid = (int)((threads + 255) / 256);
    prof_before(stream, kKBwdPre);
    bwd_preprocess_kernel<D><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(L0.o),
                                                         static_cast<const __nv_bfloat16*>(L0.dout), L0.delta,
                                                         L0.dq_acc, L0.B, L0.H, L0.Nq);
    const cudaError_t err = cudaGetLastError();
    prof_after(stream, kKBwdPre);
    if (err != cudaSuccess) return FA_ERR_CUDA;
  }
  // 2. main kernel
  CUtensorMap tq, tk, tv, tdo, tdk, tdv, tdq;
  if (!encode_bshd_map(&tq, L0.q, L0.B, L0.Nq, L0.H, D) || !encode_bshd_map(&tk, L0.k, L0.B, L0.Nk, L0.H, D) ||
      !encode_bshd_map(&tv, L0.v, L0.B, L0.Nk, L0.H, D) || !encode_bshd_map(&tdo, L0.dout, L0.B, L0.Nq, L0.H, D) ||
      !encode_bshd_map(&tdk, L0.dk, L0.B, L0.Nk, L0.H, D) || !encode_bshd_map(&tdv, L0.dv, L0.B, L0.Nk, L0.H, D) ||
      !encode_bshd_map_f32(&tdq, L0.dq_acc, L0.B, L0.Nq, L0.H, D))
    return FA_ERR_CUDA;
  BwdArgs a;
  a.lse = L0.lse;
  a.delta = L0.delta;
  a.dq_acc = L0.dq_acc;
  a.status = L0.status;
  a.B = L0.B;
  a.H = L0.H;
  a.Nq = L0.Nq;
  a.Nk = L0.Nk;
  a.causal = L0.causal;
  a.scale = L0.scale;
  a.scale_log2 = L0.scale * 1.4426950408889634f;
  a.n_kv_tiles = (L0.Nk + 127) / 128;
  a.timeout_ns = L0.timeout_ns;
  const long long grid = (long long)a.n_kv_tiles * L0.B * L0.H;
  if (grid > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  prof_before(stream, kKBwdMain);
  bwd_main_kernel<D><<<(unsigned)grid, kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, tdo, tdk, tdv, tdq, a);
  const cudaError_t err_main = cudaGetLastError();
  prof_after(stream, kKBwdMain);
  if (err_main != cudaSuccess) return FA_ERR_CUDA;
  // 3. dQ = scale * accumulator in bf16
  {
    const long long n8 = (long long)L0.B * L0.Nq * L0.H * D / 8;
    const int grid3 = (int)std::min<long long>((n8 + 255) / 256, (long long)num_sms() * 16);
    prof_before(stream, kKBwdConvert);
    bwd_convert_kernel<<<grid3, 256, 0, stream>>>(L0.dq_acc, static_cast<__nv_bfloat16*>(L0.dq), n8, L0.scale);
    const cudaError_t err = cudaGetLastError();
    prof_after(stream, kKBwdConvert);
    if (err != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

fa_status launch_bwd(const BwdLaunch& L0, cudaStream_t stream) {
  if (L0.d == 64) return launch_bwd_impl<64>(L0, stream);
  if (L0.d == 128) return launch_bwd_impl<128>(L0, stream);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
