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

constexpr int kThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-5 dS group, warps 6-9 dQ group
constexpr uint32_t kTmemCols = 512;

template <int D>
struct BwdLayout {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 16384;
  static constexpr int kQStages = (D == 64) ? 2 : 1;
  static constexpr int kDsBufs = (D == 64) ? 2 : 1;
  static constexpr int kDsBytes = 2 * 16384;  // [half][128 keys][64 queries] bf16, 128-byte swizzle
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;
  static constexpr int kOffDO = kOffQ + kQStages * kTileBytes;
  static constexpr int kOffDS = kOffDO + kQStages * kTileBytes;
  static constexpr int kOffStat = kOffDS + kDsBufs * kDsBytes;  // per dS warp: lse2[128], D[128]
  static constexpr int kOffBar = kOffStat + 4 * 2 * 128 * 4;
  // kv_full, q_full[QS], q_empty[QS], s_full[2], p_full[2], ds_free[DSB], dq_full, dq_empty, dkv_done, epi
  static constexpr int kNumBars = 1 + 2 * kQStages + 4 + kDsBufs + 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;
  // tensor memory columns
  static constexpr uint32_t kTmSt = 0;      // S^T halves at 0 and 64 (P^T bf16 written over them)
  static constexpr uint32_t kTmDPt = 128;   // dP^T halves at 128 and 192
  static constexpr uint32_t kTmDV = 256;
  static constexpr uint32_t kTmDK = 256 + D;
  static constexpr uint32_t kTmDQ = (D == 64) ? 384 : 128;  // d = 128 reuses the dP^T columns
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

// S^T half = K . Q_half^T   (M = 128 keys, N = 64 queries, K = D), both K-major.
template <int D>
__device__ __forceinline__ void issue_kq(uint32_t d_tmem, uint32_t k_smem, uint32_t q_half_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
    umma_ss(d_tmem, sdesc_sw128(k_smem + off, 16, 1024), sdesc_sw128(q_half_smem + off, 16, 1024), idesc,
            kk > 0 ? 1u : 0u);
  }
}

// acc (+)= A . B_half where B_half is 64 rows (queries) x D, read MN-major (N = D).
// A is either in tensor memory (P^T) or shared memory K-major (dS^T).
template <int D, bool kAFromTmem>
__device__ __forceinline__ void issue_acc_half(uint32_t acc_tmem, uint32_t a, uint32_t b_half_smem, bool first) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint64_t bdesc = sdesc_sw128(b_half_smem + kk * 2048, 16384, 1024);
    const uint32_t acc = (first && kk == 0) ? 0u : 1u;
    if (kAFromTmem)
      umma_ts(acc_tmem, a + kk * 8, bdesc, idesc, acc);
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                    const BwdArgs a) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
  if (a.causal) {
    const int q_lo = max(0, j * 128 - (a.Nk - a.Nq));
    i_first = q_lo >> 7;
  }
  const int n_iters = n_qtiles - i_first;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv_full, 1);
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar_q_full + s, 1);
      mbar_init(bar_q_empty + s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full + t, 1);
      mbar_init(bar_p_full + t, 128);
    }
    for (int s = 0; s < L::kDsBufs; ++s) mbar_init(bar_ds_free + s, 1);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_empty, 128);
    mbar_init(bar_dkv_done, 1);
    mbar_init(bar_epi, 128);
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

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_kv_full, 2 * L::kTileBytes);
      for (int bx = 0; bx < L::kBoxes; ++bx) {
        tma_load_4d(smem + L::kOffK + bx * L::kBoxBytes, &tmK, bar_kv_full, bx * 64, h, j * 128, b);
        tma_load_4d(smem + L::kOffV + bx * L::kBoxBytes, &tmV, bar_kv_full, bx * 64, h, j * 128, b);
      }
      for (int it = 0; it < n_iters; ++it) {
        const int st = it % L::kQStages;
        if (!mbar_wait(bar_q_empty + st, ((it / L::kQStages) & 1) ^ 1, a.timeout_ns) || *abort_flag) {
          bwd_timeout(a.status, abort_flag);
          break;
        }
        const int row = (i_first + it) * 128;
        mbar_arrive_expect_tx(bar_q_full + st, 2 * L::kTileBytes);
        for (int bx = 0; bx < L::kBoxes; ++bx) {
          tma_load_4d(smem + L::kOffQ + st * L::kTileBytes + bx * L::kBoxBytes, &tmQ, bar_q_full + st, bx * 64, h,
                      row, b);
          tma_load_4d(smem + L::kOffDO + st * L::kTileBytes + bx * L::kBoxBytes, &tmDO, bar_q_full + st, bx * 64,
                      h, row, b);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar_kv_full, 0, a.timeout_ns);
      if (!ok) bwd_timeout(a.status, abort_flag);
      tc_fence_after();
      const uint32_t k_s = sbase + L::kOffK, v_s = sbase + L::kOffV;
      for (int it = 0; it < n_iters && ok; ++it) {
        const int st = it % L::kQStages;
        const uint32_t q_s = sbase + L::kOffQ + st * L::kTileBytes;
        const uint32_t do_s = sbase + L::kOffDO + st * L::kTileBytes;
        const uint32_t ds_s = sbase + L::kOffDS + (it % L::kDsBufs) * L::kDsBytes;
        if (!mbar_wait(bar_q_full + st, (it / L::kQStages) & 1, a.timeout_ns) || *abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (D == 128 && it > 0) {  // dP^T overwrites the previous dQ tile: wait until it was read
          if (!mbar_wait(bar_dq_empty, (it - 1) & 1, a.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          issue_kq<D>(tmem + L::kTmSt + hf * 64, k_s, q_s + hf * 8192);
          issue_kq<D>(tmem + L::kTmDPt + hf * 64, v_s, do_s + hf * 8192);
          umma_commit(bar_s_full + hf);
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (!mbar_wait(bar_p_full + hf, it & 1, a.timeout_ns) || *abort_flag) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool first = (it == 0 && hf == 0);
          issue_acc_half<D, true>(tmem + L::kTmDV, tmem + L::kTmSt + hf * 64, do_s + hf * 8192, first);
          issue_acc_half<D, false>(tmem + L::kTmDK, ds_s + hf * 16384, q_s + hf * 8192, first);
        }
        if (!ok) break;
        if (D == 64 && it > 0) {  // the previous dQ tile must have left tensor memory
          if (!mbar_wait(bar_dq_empty, (it - 1) & 1, a.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        issue_dq<D>(tmem + L::kTmDQ, ds_s, k_s);
        umma_commit(bar_dq_full);
        umma_commit(bar_ds_free + (it % L::kDsBufs));
        umma_commit(bar_q_empty + st);
      }
      if (!ok) bwd_timeout(a.status, abort_flag);
      umma_commit(bar_dkv_done);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------------ dS group (thread = key)
    const uint32_t quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int key = j * 128 + r;
    const uint32_t lane_field = (quarter * 32) << 16;
    const int gw = warp - 2;  // 0..3
    float* stat = reinterpret_cast<float*>(smem + L::kOffStat) + gw * 256;  // lse2[128], D[128]
    const bool key_ok = key < a.Nk;
    const int qmin = a.causal ? key - (a.Nk - a.Nq) : INT_MIN;  // first query that sees this key
    const size_t stat_row = ((size_t)b * a.H + h) * a.Nq;
    bool ok = true;
    for (int it = 0; it < n_iters && ok; ++it) {
      const int q0 = (i_first + it) * 128;
      // stage this query tile's lse (log2 units) and D for this warp
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = lane + 32 * e;
        const int q = q0 + c;
        float l2 = INFINITY, dd = 0.f;
        if (q < a.Nq) {
          const float lse = a.lse[stat_row + q];
          l2 = (lse == -INFINITY) ? INFINITY : lse * 1.4426950408889634f;
          dd = a.delta[stat_row + q];
        }
        stat[c] = l2;
        stat[128 + c] = dd;
      }
      __syncwarp();
      // the dS buffer of this iteration must no longer be read by an earlier dQ MMA
      if (!warp_wait_b(bar_ds_free + (it % L::kDsBufs), ((it / L::kDsBufs) & 1) ^ 1, a.timeout_ns) || *abort_flag) {
        ok = false;
        break;
      }
      const uint32_t ds_u32 = sbase + L::kOffDS + (it % L::kDsBufs) * L::kDsBytes;
      // masking is needed when the tile crosses the causal diagonal or the key tail
      const bool tile_mask = (j * 128 + 128 > a.Nk) || (a.causal && (j * 128 + 127 - (a.Nk - a.Nq) > q0));
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        if (!warp_wait_b(bar_s_full + hf, it & 1, a.timeout_ns) || *abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[2][32], dp[2][32];
        tmem_ld32(tmem + lane_field + L::kTmSt + hf * 64, s[0]);
        tmem_ld32(tmem + lane_field + L::kTmSt + hf * 64 + 32, s[1]);
        tmem_ld32(tmem + lane_field + L::kTmDPt + hf * 64, dp[0]);
        tmem_ld32(tmem + lane_field + L::kTmDPt + hf * 64 + 32, dp[1]);
        tmem_ld_wait(s[0]);
        reg_pin(s[1]);
        reg_pin(dp[0]);
        reg_pin(dp[1]);
        const float* l2v = stat + hf * 64;
        const float* dv = stat + 128 + hf * 64;
        const int qh = q0 + hf * 64;
        uint32_t pk[32];
        uint32_t dk4[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float p0 = ex2(fmaf(__uint_as_float(s[c >> 5][c & 31]), a.scale_log2, -l2v[c]));
          float p1 = ex2(fmaf(__uint_as_float(s[c >> 5][(c & 31) + 1]), a.scale_log2, -l2v[c + 1]));
          if (tile_mask) {
            if (!key_ok || qh + c < qmin) p0 = 0.f;
            if (!key_ok || qh + c + 1 < qmin) p1 = 0.f;
          }
          const float ds0 = p0 * (__uint_as_float(dp[c >> 5][c & 31]) - dv[c]);
          const float ds1 = p1 * (__uint_as_float(dp[c >> 5][(c & 31) + 1]) - dv[c + 1]);
          pk[c >> 1] = pack_bf16x2(p0, p1);
          dk4[c >> 1] = pack_bf16x2(ds0, ds1);
        }
        tmem_st32(tmem + lane_field + L::kTmSt + hf * 64, pk);  // P^T, bf16 pairs, over S^T
        // dS^T row of this key: 64 queries = 8 chunks of 16 bytes, 128-byte swizzle
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint32_t addr = ds_u32 + hf * 16384 + r * 128 + ((c8 ^ (r & 7)) << 4);
          st_shared_v4(addr, dk4[c8 * 4 + 0], dk4[c8 * 4 + 1], dk4[c8 * 4 + 2], dk4[c8 * 4 + 3]);
        }
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p_full + hf);
      }
      __syncwarp();
    }
    // ---------------------------------------------------------------- dK / dV epilogue
    if (ok && warp_wait_b(bar_dkv_done, 0, a.timeout_ns) && !*abort_flag) {
      tc_fence_after();
      // stage dK in the first Q slot and dV in the first dO slot (both idle now)
      const uint32_t dk_s = sbase + L::kOffQ, dv_s = sbase + L::kOffDO;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = tmem + lane_field + (which == 0 ? L::kTmDK : L::kTmDV);
        const uint32_t dst = which == 0 ? dk_s : dv_s;
        const float mul = which == 0 ? a.scale : 1.f;
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
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_epi);
      if (warp == 2 && lane == 0) {
        if (mbar_wait(bar_epi, 0, a.timeout_ns)) {
          for (int bx = 0; bx < L::kBoxes; ++bx) {
            tma_store_4d(&tmDK, smem + L::kOffQ + bx * L::kBoxBytes, bx * 64, h, j * 128, b);
            tma_store_4d(&tmDV, smem + L::kOffDO + bx * L::kBoxBytes, bx * 64, h, j * 128, b);
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
  } else {
    // ------------------------------------------------------------------ dQ group (thread = query)
    const uint32_t quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_field = (quarter * 32) << 16;
    for (int it = 0; it < n_iters; ++it) {
      if (!warp_wait_b(bar_dq_full, it & 1, a.timeout_ns) || *abort_flag) {
        if (lane == 0) bwd_timeout(a.status, abort_flag);
        break;
      }
      tc_fence_after();
      uint32_t g[D / 32][32];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tmem + lane_field + L::kTmDQ + cc * 32, g[cc]);
      tmem_ld_wait(g[0]);
#pragma unroll
      for (int cc = 1; cc < D / 32; ++cc) reg_pin(g[cc]);
      tc_fence_before();
      mbar_arrive(bar_dq_empty);
      const int q = (i_first + it) * 128 + r;
      if (q < a.Nq) {
        float* dst = a.dq_acc + (((size_t)b * a.Nq + q) * a.H + h) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc)
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            red_add_v4(dst + cc * 32 + e, __uint_as_float(g[cc][e]), __uint_as_float(g[cc][e + 1]),
                       __uint_as_float(g[cc][e + 2]), __uint_as_float(g[cc][e + 3]));
      }
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
  CUtensorMap tq, tk, tv, tdo, tdk, tdv;
  if (!encode_bshd_map(&tq, L0.q, L0.B, L0.Nq, L0.H, D) || !encode_bshd_map(&tk, L0.k, L0.B, L0.Nk, L0.H, D) ||
      !encode_bshd_map(&tv, L0.v, L0.B, L0.Nk, L0.H, D) || !encode_bshd_map(&tdo, L0.dout, L0.B, L0.Nq, L0.H, D) ||
      !encode_bshd_map(&tdk, L0.dk, L0.B, L0.Nk, L0.H, D) || !encode_bshd_map(&tdv, L0.dv, L0.B, L0.Nk, L0.H, D))
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
  bwd_main_kernel<D><<<(unsigned)grid, kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, tdo, tdk, tdv, a);
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
