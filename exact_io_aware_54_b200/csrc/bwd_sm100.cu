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
// Kernels:
//   1. preprocess: D_i = dO_i . O_i (fp32) and a zeroed fp32 dQ accumulator;
//   2. main (tcgen05): K_j and V_j of a 128-key tile stay on chip while the 128-row
//      query tiles that can see them (from the causal diagonal onward) stream by.
//      Per query tile i:
//        S^T = K Q_i^T, dP^T = V dO_i^T       (M = 128 keys, N = 128 queries)
//        dS warps: P^T (bf16) into tensor memory, dS into a swizzled shared-
//                  memory tile (read K-major for dK and MN-major for dQ)
//        dV += P^T dO_i (P^T from tensor memory), dK += dS^T Q_i
//        dQ_i = dS K, added to the fp32 accumulator with vector reductions
//      tcgen05.mma costs about 44 cycles per instruction for any N <= 64, so the
//      score MMAs use the full N = 128.
//      d = 64, bwd_pipe_kernel: persistent, with the score MMAs, the dS warps, the
//        gradient MMAs and the dQ drain running as concurrent stages (below).
//      d = 128, bwd_main_kernel: one CTA per (b, h, key tile); the stages of a
//        query tile run one after another (tensor memory has no room for a second
//        S^T / dP^T), and the dQ tile reuses the dP^T columns.
//   3. convert: dQ = bf16(scale * accumulator).
#include "fa_internal.h"
#include "philox.cuh"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr int kThreads = 320;  // d = 128 kernel: warp 0 TMA + stats, warp 1 MMA, warps 2-9 dS warps
constexpr uint32_t kTmemCols = 512;

// Shared and tensor memory of the d = 128 kernel.
template <int D>
struct BwdLayout {
  static_assert(D == 128, "d = 64 uses PipeLayout");
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 16384;
  static constexpr int kQStages = 2;  // query tiles prefetched ahead
  static constexpr int kDsBufs = 1;
  static constexpr int kDsBytes = 2 * 16384;  // [64-query atom][128 keys][64 queries] bf16, 128-byte swizzle
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;
  static constexpr int kOffDO = kOffQ + kQStages * kTileBytes;
  static constexpr int kOffDS = kOffDO + kQStages * kTileBytes;
  static constexpr int kOffStat = kOffDS + kDsBufs * kDsBytes;  // per stage: -lse2[128], -D[128]
  static constexpr int kOffBar = kOffStat + kQStages * 2 * 128 * 4;
  // kv_full, q_full[QS], q_empty[QS], s_full, p_full, ds_free[DSB], dq_full, dq_empty, dkv_done, epi,
  // dp_full, ds_full
  static constexpr int kNumBars = 1 + 2 * kQStages + 2 + kDsBufs + 4 + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64;
  // Tensor memory columns: K, V and dS^T are read from shared memory, and the dQ
  // tile goes over the dP^T columns (drained before the next dP^T).
  static constexpr uint32_t kTmSt = 0;     // S^T, P^T bf16 over it
  static constexpr uint32_t kTmDPt = 128;  // dP^T
  static constexpr uint32_t kTmDV = 256;
  static constexpr uint32_t kTmDK = 256 + D;
  static constexpr uint32_t kTmDQ = kTmDPt;
  static_assert(kTmDK + D <= kTmemCols, "tensor memory budget");
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
  uint4* dk;  // [B, Nk, H, D] bf16, written directly by the d = 64 kernel
  uint4* dv;
  // variable-length batch (cu_q != nullptr): the sequences are packed along the
  // token axis of one batch element ([total, H, D]); Nq, Nk are the longest
  // sequence's lengths.  stat_n is the row length of lse and D ([B, H, stat_n]:
  // Nq when dense, total_q when packed).
  const int32_t* cu_q;
  const int32_t* cu_k;
  int total_q, total_k;
  int stat_n;
  // key-padding mask (null: none): [B, km_words] bits, bit j % 32 of word j / 32 set
  // when key j of the batch element takes part
  const uint32_t* key_mask;
  int km_words;
  // dropout (drop_t = 0: none), the forward's: keep when the 16-bit draw >= drop_t
  uint32_t drop_t;
  float drop_scale;
  uint32_t seed_lo, seed_hi;
  // block-sparse mask (null: dense): [H, nqb, nkb] bytes over (128-row query tile,
  // 128-key tile); 0 skips the block
  const uint8_t* block_mask;
  int nqb, nkb;
  int causal_delta;  // as for the forward: query i sees key j iff j <= i + (lk - lq) + causal_delta
};

// Where one dS block's dropout draws come from: its key, head and batch element.
struct DropCtx {
  uint32_t t;
  float scale;
  uint32_t seed_lo, seed_hi;
  int key, h, b;
};

// Whether in-range key `key` of batch element b takes part (always without a mask).
__device__ __forceinline__ bool key_attended(const BwdArgs& a, int b, int key) {
  if (a.key_mask == nullptr) return true;
  return (__ldg(a.key_mask + (size_t)b * a.km_words + (key >> 5)) >> (key & 31)) & 1u;
}


// Query tile i and key tile j of head h form a computed block (always in the dense
// instantiation).
template <bool kSparse>
__device__ __forceinline__ bool bwd_block_kept(const BwdArgs& a, int h, int i, int j) {
  if constexpr (!kSparse) return true;
  return __ldg(a.block_mask + ((size_t)h * a.nqb + i) * a.nkb + j) != 0;
}
// The first query tile >= i that key tile j of head h keeps (end when none; i itself
// in the dense instantiation).
template <bool kSparse>
__device__ __forceinline__ int next_kept_q(const BwdArgs& a, int h, int j, int i, int end) {
  if constexpr (kSparse) {
    while (i < end && !bwd_block_kept<true>(a, h, i, j)) ++i;
  }
  return i;
}

// Where sequence b lives.  Dense: batch element b of the [B, N, H, D] tensors.
// Packed: rows cu[b] .. cu[b + 1] - 1 of batch element 0.  tq / tk are the first
// query / key row along N, tb the batch coordinate; global token rows are
// tb * Nq + tq + i (queries) and tb * Nk + tk + j (keys).  lq = -1 marks offsets that
// do not fit the buffers (the sequence is skipped and the call reports a bad
// argument).
struct BwdSeq {
  int lq, lk, tq, tk, tb;
};
__device__ __forceinline__ BwdSeq bwd_seq(const BwdArgs& a, int b) {
  BwdSeq s;
  if (a.cu_q == nullptr) {
    s.lq = a.Nq;
    s.lk = a.Nk;
    s.tq = 0;
    s.tk = 0;
    s.tb = b;
    return s;
  }
  const long long q0 = a.cu_q[b], q1 = a.cu_q[b + 1], k0 = a.cu_k[b], k1 = a.cu_k[b + 1];
  const long long lq = min(q1 - q0, (long long)a.Nq), lk = min(k1 - k0, (long long)a.Nk);
  s.tq = (int)q0;
  s.tk = (int)k0;
  s.tb = 0;
  s.lq = (int)lq;
  s.lk = (int)lk;
  if (q0 < 0 || k0 < 0 || lq < 0 || lk < 0 || q0 + lq > a.total_q || k0 + lk > a.total_k) s.lq = -1;
  return s;
}

// dK = dV = 0 for the keys of a tile that no query sees (a packed sequence with
// keys but no queries): threads tid = 0 .. nthreads - 1 of the caller, 16-byte stores.
// Heads whose key tiles the d = 128 kernel runs together (its grid order).
constexpr int kHeadGroup = 16;

template <int D>
__device__ __forceinline__ void store_zero_dkv(const BwdArgs& a, const BwdSeq& s, int j, int h, int tid,
                                               int nthreads) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  for (int idx = tid; idx < 2 * 128 * kChunks; idx += nthreads) {
    const int c = idx % kChunks, row = (idx / kChunks) % 128, which = idx / (128 * kChunks);
    const int key = j * 128 + row;
    if (key < s.lk)
      (which == 0 ? a.dk : a.dv)[((size_t)((long long)s.tb * a.Nk + s.tk + key) * a.H + h) * kChunks + c] =
          make_uint4(0u, 0u, 0u, 0u);
  }
}

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

// X^T = A . B^T for one query tile (M = 128 keys, N = 128 queries, K = D): S^T = K Q^T
// or dP^T = V dO^T.  A is in tensor memory (bf16 pairs) when kAT, else K-major smem;
// B is the query-side tile, K-major smem.  Offsets in 16-byte units.
template <int D, bool kAT>
__device__ __forceinline__ void issue_scores(uint32_t d_tmem, uint32_t a_tmem, SDesc a_smem, SDesc b) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * 1024 + (kk & 3) * 2;
    if (kAT)
      umma_ts(d_tmem, a_tmem + kk * 8, sdesc_at(b, off), idesc, kk > 0 ? 1u : 0u);
    else
      umma_ss(d_tmem, sdesc_at(a_smem, off), sdesc_at(b, off), idesc, kk > 0 ? 1u : 0u);
  }
}

// acc (+)= X^T . B with X^T = P^T or dS^T (M = 128 keys, K = 128 queries) and B the
// query tile (128 queries x D) read MN-major.  In tensor memory (kAT) the dS warp
// group g keeps its 64 queries as bf16 pairs over the first 32 of its 64 columns:
// queries 16kk..16kk+15 sit at column (kk / 4) * 64 + (kk % 4) * 8.  From smem, X^T
// is the K-major dS^T tile.
template <int D, bool kAT>
__device__ __forceinline__ void issue_acc(uint32_t acc_tmem, uint32_t a_tmem, SDesc a_smem, SDesc b, bool first) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint64_t bdesc = sdesc_at(b, kk * 128);
    const uint32_t acc = (first && kk == 0) ? 0u : 1u;
    if (kAT)
      umma_ts(acc_tmem, a_tmem + (kk >> 2) * 64 + (kk & 3) * 8, bdesc, idesc, acc);
    else
      umma_ss(acc_tmem, sdesc_at(a_smem, (kk >> 2) * 1024 + (kk & 3) * 2), bdesc, idesc, acc);
  }
}

// dQ tile = dS . K  (M = 128 queries, N = D, K = 128 keys); dS and K both MN-major.
template <int D>
__device__ __forceinline__ void issue_dq(uint32_t dq_tmem, SDesc ds, SDesc k) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, true, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    umma_ss(dq_tmem, sdesc_at(ds, kk * 128), sdesc_at(k, kk * 128), idesc, kk > 0 ? 1u : 0u);
}

// P and dS for one key row and kN consecutive queries:
//   p = exp2(s * scale_log2 - lse2_q),  ds = p * (dp - D_q)
// packed to bf16 pairs.  `stat` holds -lse2 (128 floats) then -D (128 floats) of
// the query tile, already offset to the first query.  With kMask, queries before
// `qrel_min` (relative to the first query) and all queries of an out-of-range key
// get p = 0.  With kDrop, z = 0 or drop_scale per (query, key) from the dropout
// draws (philox.cuh), q0 the first query: P^T goes out as p z (the dV operand) and
// ds = p (z dp - D).
template <int kN, bool kMask, bool kDrop = false>
__device__ __forceinline__ void ds_block(const uint32_t (&sv)[kN], const uint32_t (&dp)[kN], uint32_t stat,
                                         float scale_log2, bool key_ok, int qrel_min, uint32_t (&pk)[kN / 2],
                                         uint32_t (&dsk)[kN / 2], const DropCtx* drop = nullptr, int q0 = 0) {
  const float2 sc2 = make_float2(scale_log2, scale_log2);
  // Dropout keep bits of this key for queries q0 .. q0 + kN - 1 (bit c).  One Philox
  // call covers 4 queries x 2 keys and keys 2k, 2k + 1 sit on neighbouring lanes:
  // each lane makes every other call of the pair and sends its neighbour the bits
  // of the neighbour's key.
  uint32_t keep = 0u;
  if constexpr (kDrop) {
    const uint32_t odd = (uint32_t)drop->key & 1u;
    uint32_t mine = 0u, theirs = 0u;
#pragma unroll
    for (int g = 0; g < kN / 4; g += 2) {
      const int gm = g + (int)odd;  // the query group this lane draws
      const uint4 w = philox4x32_10(
          make_uint4((uint32_t)drop->key >> 1, (uint32_t)(q0 + 4 * gm) >> 2, (uint32_t)drop->h, (uint32_t)drop->b),
          drop->seed_lo, drop->seed_hi);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = ws[e] & 0xFFFFu, hi = ws[e] >> 16;  // even key, odd key
        mine |= ((odd ? hi : lo) >= drop->t ? 1u : 0u) << (4 * gm + e);
        theirs |= ((odd ? lo : hi) >= drop->t ? 1u : 0u) << (4 * gm + e);
      }
    }
    keep = mine | __shfl_xor_sync(0xffffffffu, theirs, 1);
  }
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
    const float2 dp0 = make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1]));
    const float2 dp1 = make_float2(__uint_as_float(dp[c + 2]), __uint_as_float(dp[c + 3]));
    if constexpr (kDrop) {
      // queries q0 + c .. q0 + c + 3
      const uint32_t kq = keep >> c;
      const float2 z0 = make_float2((kq & 1u) ? drop->scale : 0.f, (kq & 2u) ? drop->scale : 0.f);
      const float2 z1 = make_float2((kq & 4u) ? drop->scale : 0.f, (kq & 8u) ? drop->scale : 0.f);
      const float2 d0 = fmul2(p0, ffma2(dp0, z0, make_float2(nd.x, nd.y)));
      const float2 d1 = fmul2(p1, ffma2(dp1, z1, make_float2(nd.z, nd.w)));
      const float2 pz0 = fmul2(p0, z0), pz1 = fmul2(p1, z1);
      pk[c / 2] = pack_bf16x2(pz0.x, pz0.y);
      pk[c / 2 + 1] = pack_bf16x2(pz1.x, pz1.y);
      dsk[c / 2] = pack_bf16x2(d0.x, d0.y);
      dsk[c / 2 + 1] = pack_bf16x2(d1.x, d1.y);
    } else {
      const float2 t0 = fadd2(dp0, make_float2(nd.x, nd.y));
      const float2 t1 = fadd2(dp1, make_float2(nd.z, nd.w));
      const float2 d0 = fmul2(p0, t0), d1 = fmul2(p1, t1);
      pk[c / 2] = pack_bf16x2(p0.x, p0.y);
      pk[c / 2 + 1] = pack_bf16x2(p1.x, p1.y);
      dsk[c / 2] = pack_bf16x2(d0.x, d0.y);
      dsk[c / 2 + 1] = pack_bf16x2(d1.x, d1.y);
    }
  }
}

// The same work as ds_block in two halves, for the d = 128 kernel, whose dP^T comes
// after the next tile's scores.  p_block: P for one key row and kN queries, left
// in `v` as fp32 (the S^T bits are overwritten), packed to bf16 pairs in pk (p z
// with dropout, the keep bits in `keep`).
template <int kN, bool kMask, bool kDrop = false>
__device__ __forceinline__ void p_block(uint32_t (&v)[kN], uint32_t stat, float scale_log2, bool key_ok,
                                        int qrel_min, uint32_t (&pk)[kN / 2], uint32_t& keep,
                                        const DropCtx* drop = nullptr, int q0 = 0) {
  const float2 sc2 = make_float2(scale_log2, scale_log2);
  keep = 0u;
  if constexpr (kDrop) {
    const uint32_t odd = (uint32_t)drop->key & 1u;
    uint32_t mine = 0u, theirs = 0u;
#pragma unroll
    for (int g = 0; g < kN / 4; g += 2) {
      const int gm = g + (int)odd;
      const uint4 w = philox4x32_10(
          make_uint4((uint32_t)drop->key >> 1, (uint32_t)(q0 + 4 * gm) >> 2, (uint32_t)drop->h, (uint32_t)drop->b),
          drop->seed_lo, drop->seed_hi);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = ws[e] & 0xFFFFu, hi = ws[e] >> 16;
        mine |= ((odd ? hi : lo) >= drop->t ? 1u : 0u) << (4 * gm + e);
        theirs |= ((odd ? lo : hi) >= drop->t ? 1u : 0u) << (4 * gm + e);
      }
    }
    keep = mine | __shfl_xor_sync(0xffffffffu, theirs, 1);
  }
#pragma unroll
  for (int c = 0; c < kN; c += 4) {
    const float4 nl = ld_shared_f4(stat + c * 4);
    const float2 x0 = ffma2(make_float2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sc2,
                            make_float2(nl.x, nl.y));
    const float2 x1 = ffma2(make_float2(__uint_as_float(v[c + 2]), __uint_as_float(v[c + 3])), sc2,
                            make_float2(nl.z, nl.w));
    float2 p0 = make_float2(ex2(x0.x), ex2(x0.y));
    float2 p1 = make_float2(ex2(x1.x), ex2(x1.y));
    if (kMask) {
      if (!key_ok || c + 0 < qrel_min) p0.x = 0.f;
      if (!key_ok || c + 1 < qrel_min) p0.y = 0.f;
      if (!key_ok || c + 2 < qrel_min) p1.x = 0.f;
      if (!key_ok || c + 3 < qrel_min) p1.y = 0.f;
    }
    v[c] = __float_as_uint(p0.x);
    v[c + 1] = __float_as_uint(p0.y);
    v[c + 2] = __float_as_uint(p1.x);
    v[c + 3] = __float_as_uint(p1.y);
    if constexpr (kDrop) {
      const uint32_t kq = keep >> c;
      const float z0 = (kq & 1u) ? drop->scale : 0.f, z1 = (kq & 2u) ? drop->scale : 0.f;
      const float z2 = (kq & 4u) ? drop->scale : 0.f, z3 = (kq & 8u) ? drop->scale : 0.f;
      pk[c / 2] = pack_bf16x2(p0.x * z0, p0.y * z1);
      pk[c / 2 + 1] = pack_bf16x2(p1.x * z2, p1.y * z3);
    } else {
      pk[c / 2] = pack_bf16x2(p0.x, p0.y);
      pk[c / 2 + 1] = pack_bf16x2(p1.x, p1.y);
    }
  }
}

// ds = p (dp - D), or p (z dp - D) with dropout, from p_block's fp32 p; `stat` as for
// p_block (-D sits 512 bytes after -lse2).
template <int kN, bool kDrop = false>
__device__ __forceinline__ void ds_from_p(const uint32_t (&pv)[kN], const uint32_t (&dp)[kN], uint32_t stat,
                                          uint32_t keep, float drop_scale, uint32_t (&dsk)[kN / 2]) {
#pragma unroll
  for (int c = 0; c < kN; c += 4) {
    const float4 nd = ld_shared_f4(stat + 512 + c * 4);
    const float2 p0 = make_float2(__uint_as_float(pv[c]), __uint_as_float(pv[c + 1]));
    const float2 p1 = make_float2(__uint_as_float(pv[c + 2]), __uint_as_float(pv[c + 3]));
    const float2 dp0 = make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1]));
    const float2 dp1 = make_float2(__uint_as_float(dp[c + 2]), __uint_as_float(dp[c + 3]));
    float2 d0, d1;
    if constexpr (kDrop) {
      const uint32_t kq = keep >> c;
      const float2 z0 = make_float2((kq & 1u) ? drop_scale : 0.f, (kq & 2u) ? drop_scale : 0.f);
      const float2 z1 = make_float2((kq & 4u) ? drop_scale : 0.f, (kq & 8u) ? drop_scale : 0.f);
      d0 = fmul2(p0, ffma2(dp0, z0, make_float2(nd.x, nd.y)));
      d1 = fmul2(p1, ffma2(dp1, z1, make_float2(nd.z, nd.w)));
    } else {
      d0 = fmul2(p0, fadd2(dp0, make_float2(nd.x, nd.y)));
      d1 = fmul2(p1, fadd2(dp1, make_float2(nd.z, nd.w)));
    }
    dsk[c / 2] = pack_bf16x2(d0.x, d0.y);
    dsk[c / 2 + 1] = pack_bf16x2(d1.x, d1.y);
  }
}

// kDrop: dropout; kSparse: block-sparse (separate instantiations, so the plain
// kernel is unchanged)
template <int D, bool kDrop, bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                    const BwdArgs a) {
  using L = BwdLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* bar_kv_full = bars;
  uint64_t* bar_q_full = bars + 1;
  uint64_t* bar_q_empty = bar_q_full + L::kQStages;
  uint64_t* bar_s_full = bar_q_empty + L::kQStages;
  uint64_t* bar_p_full = bar_s_full + 1;
  uint64_t* bar_ds_free = bar_p_full + 1;
  uint64_t* bar_dq_full = bar_ds_free + L::kDsBufs;
  uint64_t* bar_dq_empty = bar_dq_full + 1;
  uint64_t* bar_dkv_done = bar_dq_empty + 1;
  uint64_t* bar_epi = bar_dkv_done + 1;
  // s_full: S^T of a tile is ready; p_full: its P^T is in tensor memory (dV may run);
  // dp_full: its dP^T is ready; ds_full: its dS is in shared memory (dK, dQ may run)
  uint64_t* bar_dp_full = bar_epi + 1;
  uint64_t* bar_ds_full = bar_dp_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 8);

  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t sbase = smem_u32(smem);

  // work: key tile j of head (b, h).  Heads go in groups of kHeadGroup, and the key
  // tiles of one group's heads run together, heavy (early) key tiles first under the
  // causal mask: the fp32 dQ rows that a head's key tiles add to then stay in L2
  // between them, where with every head's key tile j before any key tile j + 1 they
  // were evicted in between (long sequences moved 6.6x the ideal DRAM bytes)
  const int bh_count = a.B * a.H;
  const int gi = blockIdx.x / (a.n_kv_tiles * kHeadGroup);
  const int g0 = gi * kHeadGroup;
  const int gsz = min(kHeadGroup, bh_count - g0);
  const int in_group = blockIdx.x - gi * (a.n_kv_tiles * kHeadGroup);
  const int j = in_group / gsz;
  const int bh = g0 + (in_group - j * gsz);
  const int b = bh / a.H, h = bh - (bh / a.H) * a.H;
  const BwdSeq sq = bwd_seq(a, b);
  if (sq.lq < 0) {  // block-uniform exits, before any barrier or tensor memory
    if (threadIdx.x == 0) atomicExch(a.status, kStatusBadArg);
    return;
  }
  if (j * 128 >= sq.lk) return;  // no key of this sequence in the tile
  const int n_qtiles = (sq.lq + 127) >> 7;
  int i_first = 0;
  if (a.causal) i_first = max(0, j * 128 - (sq.lk - sq.lq + a.causal_delta)) >> 7;
  int n_iters = n_qtiles - i_first;  // >= 1 when the sequence has queries
  if constexpr (kSparse) {  // the kept query tiles only
    n_iters = 0;
    for (int i = i_first; i < n_qtiles; ++i) n_iters += bwd_block_kept<true>(a, h, i, j) ? 1 : 0;
  }
  if (n_iters <= 0) {
    store_zero_dkv<D>(a, sq, j, h, threadIdx.x, blockDim.x);
    return;
  }
  // a packed sequence's partial last key tile is stored row by row: a tile store
  // would run into the next sequence's rows
  const bool direct_dkv = a.cu_q != nullptr && j * 128 + 128 > sq.lk;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv_full, 1);
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar_q_full + s, 2);  // TMA bytes + the producer's stats
      mbar_init(bar_q_empty + s, 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_p_full, 8);  // one arrival per dS warp
    for (int s = 0; s < L::kDsBufs; ++s) mbar_init(bar_ds_free + s, 1);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_empty, 8);
    mbar_init(bar_dkv_done, 1);
    mbar_init(bar_epi, 8);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_ds_full, 8);
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
  const size_t stat_row = ((size_t)sq.tb * a.H + h) * a.stat_n + sq.tq;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer: TMA tiles + lse/D
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_kv_full, 2 * L::kTileBytes);
      for (int bx = 0; bx < L::kBoxes; ++bx) {
        tma_load_4d(smem + L::kOffK + bx * L::kBoxBytes, &tmK, bar_kv_full, bx * 64, h, sq.tk + j * 128, sq.tb);
        tma_load_4d(smem + L::kOffV + bx * L::kBoxBytes, &tmV, bar_kv_full, bx * 64, h, sq.tk + j * 128, sq.tb);
      }
    }
    int qi = next_kept_q<kSparse>(a, h, j, i_first, n_qtiles);  // query tile of step it
    for (int it = 0; it < n_iters; ++it, qi = next_kept_q<kSparse>(a, h, j, qi + 1, n_qtiles)) {
      const int st = it % L::kQStages;
      const int q0 = qi * 128;
      // -lse in log2 units (-inf for rows past Nq or with no visible key: P = 0 there)
      // and -D, negated so that the dS warps use them as addends.  The global loads
      // are issued before waiting for the stage so that their latency overlaps it.
      float nl2[4], nd[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = q0 + lane + 32 * e;
        nl2[e] = -INFINITY;
        nd[e] = 0.f;
        if (q < sq.lq) {
          const float lse = a.lse[stat_row + q];
          nl2[e] = (lse == -INFINITY) ? -INFINITY : -lse * 1.4426950408889634f;
          nd[e] = -a.delta[stat_row + q];
        }
      }
      bool ok = true;
      if (lane == 0) ok = mbar_wait(bar_q_empty + st, ((it / L::kQStages) & 1) ^ 1, a.timeout_ns) && !*abort_flag;
      if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) {
        if (lane == 0) bwd_timeout(a.status, abort_flag);
        break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar_q_full + st, 2 * L::kTileBytes);
        for (int bx = 0; bx < L::kBoxes; ++bx) {
          tma_load_4d(smem + L::kOffQ + st * L::kTileBytes + bx * L::kBoxBytes, &tmQ, bar_q_full + st, bx * 64, h,
                      sq.tq + q0, sq.tb);
          tma_load_4d(smem + L::kOffDO + st * L::kTileBytes + bx * L::kBoxBytes, &tmDO, bar_q_full + st, bx * 64,
                      h, sq.tq + q0, sq.tb);
        }
      }
      float* stat = reinterpret_cast<float*>(smem + L::kOffStat) + st * 256;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        stat[lane + 32 * e] = nl2[e];
        stat[128 + lane + 32 * e] = nd[e];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_q_full + st);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar_kv_full, 0, a.timeout_ns);
      // operand descriptors, built once; tiles are reached by 32-bit adds (16-byte units)
      const SDesc k_kmaj = sdesc_make(sbase + L::kOffK, 16, 1024), v_kmaj = sdesc_make(sbase + L::kOffV, 16, 1024);
      const SDesc k_mn = sdesc_make(sbase + L::kOffK, 16384, 1024);
      const SDesc q_kmaj = sdesc_make(sbase + L::kOffQ, 16, 1024), do_kmaj = sdesc_make(sbase + L::kOffDO, 16, 1024);
      const SDesc q_mn = sdesc_make(sbase + L::kOffQ, 16384, 1024), do_mn = sdesc_make(sbase + L::kOffDO, 16384, 1024);
      const SDesc ds_kmaj = sdesc_make(sbase + L::kOffDS, 16, 1024), ds_mn = sdesc_make(sbase + L::kOffDS, 16384, 1024);
      constexpr uint32_t kTile16 = L::kTileBytes / 16, kDs16 = L::kDsBytes / 16;
      auto at = [](SDesc d, uint32_t off16) { return SDesc{d.lo + off16, d.hi}; };
      auto wait_ok = [&](uint64_t* bar, uint32_t parity) {
        return mbar_wait(bar, parity, a.timeout_ns) && !*abort_flag;
      };
      // Per query tile `it`: dP^T (after the previous dQ has left the dP^T columns),
      // dV once P^T is written, then the next tile's S^T (it reuses the S^T columns
      // after dV has read P^T: tcgen05 operations run in issue order), and dK and dQ
      // once dS is written.  The dS warps compute the next tile's P while dK and dQ
      // run.
      if (ok && (ok = wait_ok(bar_q_full, 0))) {
        tc_fence_after();
        issue_scores<D, false>(tmem + L::kTmSt, 0u, k_kmaj, q_kmaj);
        umma_commit(bar_s_full);
      }
      for (int it = 0; it < n_iters && ok; ++it) {
        const int st = it % L::kQStages;
        if (it > 0) {
          if (!(ok = wait_ok(bar_dq_empty, (it - 1) & 1))) break;
          tc_fence_after();
        }
        issue_scores<D, false>(tmem + L::kTmDPt, 0u, v_kmaj, at(do_kmaj, st * kTile16));
        umma_commit(bar_dp_full);
        if (!(ok = wait_ok(bar_p_full, it & 1))) break;
        tc_fence_after();
        issue_acc<D, true>(tmem + L::kTmDV, tmem + L::kTmSt, ds_kmaj, at(do_mn, st * kTile16), it == 0);
        if (it + 1 < n_iters) {
          const int sn = (it + 1) % L::kQStages;
          if (!(ok = wait_ok(bar_q_full + sn, ((it + 1) / L::kQStages) & 1))) break;
          tc_fence_after();
          issue_scores<D, false>(tmem + L::kTmSt, 0u, k_kmaj, at(q_kmaj, sn * kTile16));
          umma_commit(bar_s_full);
        }
        if (!(ok = wait_ok(bar_ds_full, it & 1))) break;
        tc_fence_after();
        issue_acc<D, false>(tmem + L::kTmDK, 0u, at(ds_kmaj, (it % L::kDsBufs) * kDs16), at(q_mn, st * kTile16),
                            it == 0);
        umma_commit(bar_q_empty + st);  // Q and dO of this tile are no longer read
        issue_dq<D>(tmem + L::kTmDQ, at(ds_mn, (it % L::kDsBufs) * kDs16), k_mn);
        umma_commit(bar_dq_full);
        umma_commit(bar_ds_free + (it % L::kDsBufs));
      }
      if (!ok) bwd_timeout(a.status, abort_flag);
      umma_commit(bar_dkv_done);
    }
  } else {
    // ------------------------------------------------------------------ dS warps (thread = key)
    const uint32_t quarter = warp & 3;
    const int grp = (warp - 2) >> 2;  // column group: queries [64 grp, 64 grp + 64) of each tile
    const int r = quarter * 32 + lane;
    const int key = j * 128 + r;
    const uint32_t lane_field = (quarter * 32) << 16;
    const bool key_in = key < sq.lk;  // a row of dK / dV to write
    const bool key_ok = key_in && key_attended(a, b, key);  // and its P is not masked out
    // first query that sees this key (a sentinel far below any query when not causal;
    // qmin - qs below must not overflow)
    const int qmin = a.causal ? key - (sq.lk - sq.lq + a.causal_delta) : -(1 << 30);
    bool ok = true;

    // dQ tile of query tile `it`: this group's D/2 columns, 32 at a time, turned
    // around in this warp's 4 KB of the dS buffer (free once the dQ product has
    // completed; the next dS is written by this same warp) so that one vector
    // reduction covers four whole 128-byte rows: reductions of partial rows run at
    // about half the L2 rate
    const int rr_sub = lane >> 3, cc = lane & 7;  // read side: row 4k + rr_sub, chunk cc
    const uint32_t scratch = sbase + L::kOffDS + grp * 16384 + quarter * 4096;
    auto drain_dq = [&](int it, int q_first) -> bool {
      if (!warp_wait_b(bar_dq_full, it & 1, a.timeout_ns) || *abort_flag) return false;
      tc_fence_after();
      // both halves out of tensor memory first, so the next dP^T can start at once
      uint32_t g[2][32];
      tmem_ld32(tmem + lane_field + L::kTmDQ + grp * (D / 2), g[0]);
      tmem_ld32(tmem + lane_field + L::kTmDQ + grp * (D / 2) + 32, g[1]);
      tmem_ld_wait(g[0]);
      reg_pin(g[1]);
      tc_fence_before();
      mbar_arrive_warp(bar_dq_empty);
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(scratch + lane * 128 + ((c ^ (lane & 7)) << 4), g[pass][4 * c], g[pass][4 * c + 1],
                       g[pass][4 * c + 2], g[pass][4 * c + 3]);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int row = 4 * k + rr_sub;
          const int q = q_first + (int)quarter * 32 + row;
          const float4 v4 = ld_shared_f4(scratch + row * 128 + ((cc ^ (row & 7)) << 4));
          if (q < sq.lq)
            red_add_v4(a.dq_acc + ((size_t)((long long)sq.tb * a.Nq + sq.tq + q) * a.H + h) * D + grp * (D / 2) +
                           pass * 32 + cc * 4,
                       v4.x, v4.y, v4.z, v4.w);
        }
        __syncwarp();
      }
      return true;
    };

    // P of query tile `it` (stage st, first query q0): the group's 64 queries in two
    // chunks of 32, fp32 p kept in pv for the dS that follows, P^T (bf16) over the
    // S^T columns already read
    uint32_t pv[2][32];
    uint32_t keep[2] = {0u, 0u};
    auto p_phase = [&](int it, int q0) -> bool {
      const int st = it % L::kQStages;
      if (!warp_wait_b(bar_q_full + st, (it / L::kQStages) & 1, a.timeout_ns) ||
          !warp_wait_b(bar_s_full, it & 1, a.timeout_ns) || *abort_flag)
        return false;
      tc_fence_after();
      tmem_ld32(tmem + lane_field + L::kTmSt + 64 * grp, pv[0]);
      tmem_ld32(tmem + lane_field + L::kTmSt + 64 * grp + 32, pv[1]);
      tmem_ld_wait(pv[0]);
      reg_pin(pv[1]);
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int col = 64 * grp + 32 * ch;
        const int qs = q0 + col;
        const uint32_t stat_u32 = sbase + L::kOffStat + st * 1024 + col * 4;
        const bool tile_mask = a.key_mask != nullptr || (j * 128 + 128 > sq.lk) ||
                               (a.causal && (j * 128 + 127 - (sq.lk - sq.lq + a.causal_delta) > qs));
        uint32_t pk[16];
        if constexpr (kDrop) {
          const DropCtx dctx{a.drop_t, a.drop_scale, a.seed_lo, a.seed_hi, key, h, b};
          p_block<32, true, true>(pv[ch], stat_u32, a.scale_log2, key_ok, qmin - qs, pk, keep[ch], &dctx, qs);
        } else if (tile_mask) {
          p_block<32, true>(pv[ch], stat_u32, a.scale_log2, key_ok, qmin - qs, pk, keep[ch]);
        } else {
          p_block<32, false>(pv[ch], stat_u32, a.scale_log2, key_ok, qmin - qs, pk, keep[ch]);
        }
        tmem_st16(tmem + lane_field + L::kTmSt + 64 * grp + 16 * ch, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar_p_full);  // dV may read P^T
      return true;
    };

    // dS of query tile `it` from pv and dP^T, into the dS buffer (128-byte swizzle)
    auto ds_phase = [&](int it) -> bool {
      const int st = it % L::kQStages;
      if (!warp_wait_b(bar_ds_free + (it % L::kDsBufs), ((it / L::kDsBufs) & 1) ^ 1, a.timeout_ns) ||
          !warp_wait_b(bar_dp_full, it & 1, a.timeout_ns) || *abort_flag)
        return false;
      tc_fence_after();
      const uint32_t ds_row = sbase + L::kOffDS + (it % L::kDsBufs) * L::kDsBytes + grp * 16384 + r * 128;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int col = 64 * grp + 32 * ch;
        uint32_t dp[32];
        tmem_ld32(tmem + lane_field + L::kTmDPt + col, dp);
        tmem_ld_wait(dp);
        uint32_t dk2[16];
        ds_from_p<32, kDrop>(pv[ch], dp, sbase + L::kOffStat + st * 1024 + col * 4, keep[ch], a.drop_scale, dk2);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int chunk = 4 * ch + c4;
          st_shared_v4(ds_row + ((chunk ^ (r & 7)) << 4), dk2[4 * c4], dk2[4 * c4 + 1], dk2[4 * c4 + 2],
                       dk2[4 * c4 + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive_warp(bar_ds_full);  // dK and dQ may read dS
      return true;
    };

    int qi = next_kept_q<kSparse>(a, h, j, i_first, n_qtiles);  // query tile of step it
    ok = p_phase(0, qi * 128);
    for (int it = 0; it < n_iters && ok; ++it) {
      const int q0 = qi * 128;
      if (!(ok = ds_phase(it))) break;
      // the next tile's P while dK and dQ of this one run
      const int qn = next_kept_q<kSparse>(a, h, j, qi + 1, n_qtiles);
      if (it + 1 < n_iters && !(ok = p_phase(it + 1, qn * 128))) break;
      ok = drain_dq(it, q0);
      qi = qn;
    }
    // ---------------------------------------------------------------- dK / dV epilogue
    // group 0 stores dK (times scale) through the K tile's smem, group 1 dV through V's;
    // with direct_dkv each thread writes its key row straight to global memory
    if (ok && warp_wait_b(bar_dkv_done, 0, a.timeout_ns) && !*abort_flag) {
      tc_fence_after();
      const uint32_t src = tmem + lane_field + (grp == 0 ? L::kTmDK : L::kTmDV);
      const uint32_t dst = sbase + (grp == 0 ? L::kOffK : L::kOffV);
      uint4* gdst = (grp == 0 ? a.dk : a.dv) + ((size_t)((long long)sq.tb * a.Nk + sq.tk + key) * a.H + h) * (D / 8);
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
          const float* f = reinterpret_cast<const float*>(o) + q4 * 8;
          const uint4 w = make_uint4(pack_bf16x2(f[0] * mul, f[1] * mul), pack_bf16x2(f[2] * mul, f[3] * mul),
                                     pack_bf16x2(f[4] * mul, f[5] * mul), pack_bf16x2(f[6] * mul, f[7] * mul));
          if (!direct_dkv)
            st_shared_v4(dst + box * L::kBoxBytes + r * 128 + ((chunk ^ (r & 7)) << 4), w.x, w.y, w.z, w.w);
          else if (key_in)
            gdst[cc * 4 + q4] = w;
        }
      }
      if (!direct_dkv) {
        fence_proxy_async_smem();
        mbar_arrive_warp(bar_epi);
        if (warp == 2 && lane == 0) {
          if (mbar_wait(bar_epi, 0, a.timeout_ns)) {
            for (int bx = 0; bx < L::kBoxes; ++bx) {
              tma_store_4d(&tmDK, smem + L::kOffK + bx * L::kBoxBytes, bx * 64, h, sq.tk + j * 128, sq.tb);
              tma_store_4d(&tmDV, smem + L::kOffV + bx * L::kBoxBytes, bx * 64, h, sq.tk + j * 128, sq.tb);
            }
            bulk_commit_group();
            bulk_wait_group0();
          } else {
            bwd_timeout(a.status, abort_flag);
          }
        }
        __syncwarp();
      }
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

// ------------------------------------------------------------------------------------
// d = 64: pipelined main kernel.
//
// The dS warps copy S^T and dP^T of a query tile into registers and release both
// tensor-memory tiles at once, so the tensor core computes the next tile's scores
// while they work.  P^T goes to its own tensor-memory columns and dK reads dS^T
// from shared memory: no tensor-memory location is written by one MMA while an
// earlier MMA still reads it, so the tensor core never drains between tiles.  Four
// drain warps move each dQ tile out of tensor memory and add it to the fp32
// accumulator.  A thread holds one query row; each warp turns its 32 rows around
// in shared memory so that one vector reduction instruction covers four whole
// 128-byte rows (reductions of partial rows run at half the L2 rate).
//
// Two threads issue MMAs: one the scores S^T(i), dP^T(i) (as soon as the dS warps
// have released tile i - 1), the other the gradient products dV(i), dK(i), dQ(i)
// (as soon as tile i's P^T and dS are written).  The two streams use disjoint
// tensor-memory columns and meet only through the dS warps, so neither waits
// behind the other's back-pressured issue queue.
// dS warps:    load S^T(i), dP^T(i) -> release -> P^T(i) to TMEM, dS(i) to smem
// drain warps: dQ(i) TMEM -> registers -> release -> smem transpose -> red.global.add.v4
//
// The kernel is persistent: one CTA per SM walks the work items (key tile, b, h),
// heaviest first.  Every role counts query tiles over all its items, so the
// per-tile barriers run on one stream of phases.  K has two slots and the next
// item's K is loaded a whole item ahead; V has one slot, released after the item's
// last dP^T, so the next V loads while the last query tile is finished.  The dQ
// drain warps also write each item's dK and dV (tensor memory -> registers ->
// global memory), so the dS warps go straight on to the next item's first query
// tile (when the dS warps wrote them, they waited on the item's last gradient
// MMAs: 12% of their time, and the kernel was 3% slower).
struct PipeLayout {
  static constexpr int D = 64;
  static constexpr int kTileBytes = 128 * D * 2;  // 16 KB
  static constexpr int kQStages = 3;
  static constexpr int kDsBufs = 2;
  static constexpr int kDsBytes = 2 * 16384;  // [64-query atom][128 keys][64 queries] bf16
  // the drain warps turn dQ rows around in the first 16 KB of the dS buffer of the
  // tile they drain (its MMAs have completed; its next writer waits for them)
  static constexpr int kScratchBytes = 4 * 32 * 128;
  static constexpr int kOffK = 0;  // two slots
  static constexpr int kOffV = 2 * kTileBytes;
  static constexpr int kOffQ = 3 * kTileBytes;
  static constexpr int kOffDO = kOffQ + kQStages * kTileBytes;
  static constexpr int kOffDS = kOffDO + kQStages * kTileBytes;
  static constexpr int kOffStat = kOffDS + kDsBufs * kDsBytes;  // per stage: -lse2[128], -D[128]
  static constexpr int kOffBar = kOffStat + kQStages * 2 * 128 * 4;
  // k_full[2], k_free[2], v_full, v_free, q_full[QS], q_empty[QS], s_full, s_free, p_full,
  // pt_free, ds_free[DSB], dq_full, dq_empty, dkv_done, acc_free
  static constexpr int kNumBars = 6 + 2 * kQStages + 4 + kDsBufs + 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64;
  static constexpr uint32_t kTmSt = 0, kTmDPt = 128, kTmPt = 256, kTmDV = 320, kTmDK = 384, kTmDQ = 448;
  static_assert(kTmDQ + D <= kTmemCols, "tensor memory budget");
  static_assert(kScratchBytes <= kDsBytes, "drain scratch");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};
// warps 0-3: TMA producer, score MMA issuer, gradient MMA issuer, idle; 4-7: dQ drain;
// 8-15: dS (two column groups)
constexpr int kPipeThreads = 512;
constexpr uint32_t kPipeRegsCtl = 72, kPipeRegsDrain = 104, kPipeRegsDs = 168;
static_assert(128 * kPipeRegsCtl + 128 * kPipeRegsDrain + 256 * kPipeRegsDs <= kPipeThreads * 128,
              "register split exceeds the launch budget");

// acc (+)= X^T . B with X^T (M = 128 keys, K = 128 queries) in tensor memory as bf16
// pairs, query pair p at column p; B the query tile read MN-major.
template <int D>
__device__ __forceinline__ void issue_acc_tmem_linear(uint32_t acc_tmem, uint32_t a_tmem, SDesc b, bool first) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    umma_ts(acc_tmem, a_tmem + kk * 8, sdesc_at(b, kk * 128), idesc, (first && kk == 0) ? 0u : 1u);
}

// Work item w: key tile j = w / (B H) (small j first: under the causal mask they see
// the most query tiles), head (b, h) = w % (B H); query tiles i_first .. n_qtiles - 1.
// CTA c takes the items of its column in a snake order over rounds of gridDim.x
// items (c, 2G - 1 - c, 2G + c, ...), which pairs heavy rounds with light ones.
__device__ __forceinline__ int pipe_item_index(int k) {
  const int g = gridDim.x;
  return k * g + ((k & 1) ? (g - 1 - (int)blockIdx.x) : (int)blockIdx.x);
}
// n = number of query tiles; n = 0 for a tile of keys that no query sees (their dK
// and dV are zero), n = -1 for a tile past the sequence's last key or a sequence
// with bad offsets.  Only items with n > 0 take part in the pipeline, and the
// barrier phases of every role count those items alone.
struct PipeItem {
  int j, b, h, i_first, n;
  BwdSeq s;
};
template <bool kSparse>
__device__ __forceinline__ PipeItem pipe_item(const BwdArgs& a, int w) {
  PipeItem it;
  const int bh_count = a.B * a.H;
  // key tile j of every head, then j + 1: the heaviest causal items first
  it.j = w / bh_count;
  const int bh = w - it.j * bh_count;
  const int b = bh / a.H;
  it.b = b;
  it.h = bh - b * a.H;
  it.s = bwd_seq(a, b);
  it.i_first = 0;
  it.n = -1;
  if (it.s.lq < 0 || it.j * 128 >= it.s.lk) return it;
  const int n_qtiles = (it.s.lq + 127) >> 7;
  it.i_first = a.causal ? (max(0, it.j * 128 - (it.s.lk - it.s.lq + a.causal_delta)) >> 7) : 0;
  it.n = max(0, n_qtiles - it.i_first);  // 0: keys no query sees (dK = dV = 0)
  if constexpr (kSparse) {  // the kept query tiles only
    it.n = 0;
    for (int i = it.i_first; i < n_qtiles; ++i) it.n += bwd_block_kept<true>(a, it.h, i, it.j) ? 1 : 0;
  }
  return it;
}

// Walks the query tiles of this CTA's items (those with query tiles) in order.
template <bool kSparse>
struct PipeCursor {
  int k;   // item index of this CTA (pipe_item_index)
  int u;   // items with query tiles passed so far
  int t;   // query tile within the item (counting the item's tiles)
  int qi;  // that query tile's index (block-sparse instantiation)
  bool valid;
  PipeItem itm;
  __device__ __forceinline__ int qtile() const {
    if constexpr (kSparse) return qi;
    return itm.i_first + t;
  }
  __device__ __forceinline__ void first_q(const BwdArgs& a) {
    if constexpr (kSparse) qi = next_kept_q<true>(a, itm.h, itm.j, itm.i_first, (itm.s.lq + 127) >> 7);
  }
  // from item k on, the first item with query tiles
  __device__ __forceinline__ void seek(const BwdArgs& a, int n_items) {
    for (;; ++k) {
      const int w = pipe_item_index(k);
      valid = w < n_items;
      if (!valid) return;
      itm = pipe_item<kSparse>(a, w);
      if (itm.n > 0) {
        first_q(a);
        return;
      }
    }
  }
  __device__ __forceinline__ void start(const BwdArgs& a, int n_items) {
    k = 0;
    u = 0;
    t = 0;
    seek(a, n_items);
  }
  __device__ __forceinline__ void advance(const BwdArgs& a, int n_items) {
    if (++t < itm.n) {
      if constexpr (kSparse) qi = next_kept_q<true>(a, itm.h, itm.j, qi + 1, (itm.s.lq + 127) >> 7);
      return;
    }
    t = 0;
    ++k;
    ++u;
    seek(a, n_items);
  }
};

// -lse in log2 units (-inf for rows past Nq or with no visible key: P = 0) and -D of
// four query rows per lane, negated so that the dS warps add them.
template <bool kSparse>
__device__ __forceinline__ void pipe_load_stats(const BwdArgs& a, const PipeCursor<kSparse>& c, uint32_t lane,
                                                float (&nl2)[4], float (&nd)[4]) {
  const size_t stat_row = ((size_t)c.itm.s.tb * a.H + c.itm.h) * a.stat_n + c.itm.s.tq;
  const int q0 = c.qtile() * 128;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int q = q0 + lane + 32 * e;
    nl2[e] = -INFINITY;
    nd[e] = 0.f;
    if (q < c.itm.s.lq) {
      const float lse = a.lse[stat_row + q];
      nl2[e] = (lse == -INFINITY) ? -INFINITY : -lse * 1.4426950408889634f;
      nd[e] = -a.delta[stat_row + q];
    }
  }
}

// kDrop: dropout; kSparse: block-sparse (separate instantiations, so the plain
// kernel is unchanged)
template <bool kDrop, bool kSparse>
__global__ void __launch_bounds__(kPipeThreads, 1)
    bwd_pipe_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdArgs a) {
  using L = PipeLayout;
  constexpr int D = L::D;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* bar_k_full = bars;  // [2]
  uint64_t* bar_k_free = bars + 2;  // [2]
  uint64_t* bar_v_full = bars + 4;
  uint64_t* bar_v_free = bars + 5;
  uint64_t* bar_q_full = bars + 6;
  uint64_t* bar_q_empty = bar_q_full + L::kQStages;
  uint64_t* bar_s_full = bar_q_empty + L::kQStages;
  uint64_t* bar_s_free = bar_s_full + 1;
  uint64_t* bar_p_full = bar_s_free + 1;
  uint64_t* bar_pt_free = bar_p_full + 1;
  uint64_t* bar_ds_free = bar_pt_free + 1;
  uint64_t* bar_dq_full = bar_ds_free + L::kDsBufs;
  uint64_t* bar_dq_empty = bar_dq_full + 1;
  uint64_t* bar_dkv_done = bar_dq_empty + 1;
  uint64_t* bar_acc_free = bar_dkv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 8);

  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t sbase = smem_u32(smem);
  const int n_items = a.n_kv_tiles * a.B * a.H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_k_full + s, 1);
      mbar_init(bar_k_free + s, 1);
    }
    mbar_init(bar_v_full, 1);
    mbar_init(bar_v_free, 1);
    for (int s = 0; s < L::kQStages; ++s) {
      mbar_init(bar_q_full + s, 2);  // TMA bytes + the producer's stats
      mbar_init(bar_q_empty + s, 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_s_free, 8);  // one arrival per dS warp
    mbar_init(bar_p_full, 8);
    mbar_init(bar_pt_free, 1);
    for (int s = 0; s < L::kDsBufs; ++s) mbar_init(bar_ds_free + s, 1 + 4);  // dQ MMA + the drain warps
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_empty, 4);  // one arrival per drain warp
    mbar_init(bar_dkv_done, 1);
    mbar_init(bar_acc_free, 4);  // one arrival per drain warp
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

  if (warp < 4) {
    regs_dec<kPipeRegsCtl>();
    if (warp == 0) {
      // -------------------------------------------------------------- producer: TMA tiles + lse/D
      PipeCursor<kSparse> cur;
      cur.start(a, n_items);
      bool ok = true;
      float nl2[4], nd[4];
      if (cur.valid) {
        pipe_load_stats(a, cur, lane, nl2, nd);
        if (lane == 0) {  // the first item's K and V
          mbar_arrive_expect_tx(bar_k_full, L::kTileBytes);
          tma_load_4d(smem + L::kOffK, &tmK, bar_k_full, 0, cur.itm.h, cur.itm.s.tk + cur.itm.j * 128, cur.itm.s.tb);
          mbar_arrive_expect_tx(bar_v_full, L::kTileBytes);
          tma_load_4d(smem + L::kOffV, &tmV, bar_v_full, 0, cur.itm.h, cur.itm.s.tk + cur.itm.j * 128, cur.itm.s.tb);
        }
      }
      for (int T = 0; cur.valid && ok; ++T) {
        const int st = T % L::kQStages;
        const int q0 = cur.qtile() * 128;
        PipeCursor<kSparse> nxt = cur;
        nxt.advance(a, n_items);
        // the next tile's statistics are loaded while this tile waits for its stage
        float nl2n[4], ndn[4];
        if (nxt.valid) pipe_load_stats(a, nxt, lane, nl2n, ndn);
        bool got = true;
        if (lane == 0) got = mbar_wait(bar_q_empty + st, ((T / L::kQStages) & 1) ^ 1, a.timeout_ns) && !*abort_flag;
        if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_q_full + st, 2 * L::kTileBytes);
          tma_load_4d(smem + L::kOffQ + st * L::kTileBytes, &tmQ, bar_q_full + st, 0, cur.itm.h, cur.itm.s.tq + q0,
                      cur.itm.s.tb);
          tma_load_4d(smem + L::kOffDO + st * L::kTileBytes, &tmDO, bar_q_full + st, 0, cur.itm.h,
                      cur.itm.s.tq + q0, cur.itm.s.tb);
        }
        float* stat = reinterpret_cast<float*>(smem + L::kOffStat) + st * 256;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          stat[lane + 32 * e] = nl2[e];
          stat[128 + lane + 32 * e] = nd[e];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_q_full + st);
        if (cur.t + 1 == cur.itm.n && nxt.valid) {
          // the last query tile of item u is staged: load item u + 1's K (into the slot
          // item u - 1 used) and V (once item u's last dP^T has read it)
          const int u1 = cur.u + 1;
          if (lane == 0) {
            got = (u1 < 2 || mbar_wait(bar_k_free + (u1 & 1), ((u1 >> 1) - 1) & 1, a.timeout_ns)) && !*abort_flag;
            if (got) {
              mbar_arrive_expect_tx(bar_k_full + (u1 & 1), L::kTileBytes);
              tma_load_4d(smem + L::kOffK + (u1 & 1) * L::kTileBytes, &tmK, bar_k_full + (u1 & 1), 0, nxt.itm.h,
                          nxt.itm.s.tk + nxt.itm.j * 128, nxt.itm.s.tb);
              got = mbar_wait(bar_v_free, cur.u & 1, a.timeout_ns) && !*abort_flag;
            }
            if (got) {
              mbar_arrive_expect_tx(bar_v_full, L::kTileBytes);
              tma_load_4d(smem + L::kOffV, &tmV, bar_v_full, 0, nxt.itm.h, nxt.itm.s.tk + nxt.itm.j * 128,
                          nxt.itm.s.tb);
            }
          }
          if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0) {
            ok = false;
            break;
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          nl2[e] = nl2n[e];
          nd[e] = ndn[e];
        }
        cur = nxt;
      }
      if (!ok && lane == 0) bwd_timeout(a.status, abort_flag);
    } else if ((warp == 1 || warp == 2) && lane == 0) {
      const SDesc k_kmaj = sdesc_make(sbase + L::kOffK, 16, 1024), v_kmaj = sdesc_make(sbase + L::kOffV, 16, 1024);
      const SDesc k_mn = sdesc_make(sbase + L::kOffK, 16384, 1024);
      const SDesc q_kmaj = sdesc_make(sbase + L::kOffQ, 16, 1024), do_kmaj = sdesc_make(sbase + L::kOffDO, 16, 1024);
      const SDesc q_mn = sdesc_make(sbase + L::kOffQ, 16384, 1024), do_mn = sdesc_make(sbase + L::kOffDO, 16384, 1024);
      const SDesc ds_kmaj = sdesc_make(sbase + L::kOffDS, 16, 1024), ds_mn = sdesc_make(sbase + L::kOffDS, 16384, 1024);
      constexpr uint32_t kTile16 = L::kTileBytes / 16, kDs16 = L::kDsBytes / 16;
      auto at = [](SDesc d, uint32_t off16) { return SDesc{d.lo + off16, d.hi}; };
      bool ok = true;
      int T = 0, u = 0;
      if (warp == 1) {
        // ------------------------------------------------------------ score MMAs
        for (int k = 0, w; (w = pipe_item_index(k)) < n_items && ok; ++k) {
          const PipeItem itm = pipe_item<kSparse>(a, w);
          if (itm.n <= 0) continue;
          const int ks = u & 1;
          if (!mbar_wait(bar_k_full + ks, (u >> 1) & 1, a.timeout_ns) || !mbar_wait(bar_v_full, u & 1, a.timeout_ns) ||
              *abort_flag) {
            ok = false;
            break;
          }
          for (int t = 0; t < itm.n; ++t, ++T) {
            const int st = T % L::kQStages;
            // this tile's Q and dO; S^T / dP^T free again (the dS warps hold tile T - 1)
            if (!mbar_wait(bar_q_full + st, (T / L::kQStages) & 1, a.timeout_ns) ||
                (T > 0 && !mbar_wait(bar_s_free, (T - 1) & 1, a.timeout_ns)) || *abort_flag) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_scores<D, false>(tmem + L::kTmSt, 0u, at(k_kmaj, ks * kTile16), at(q_kmaj, st * kTile16));
            issue_scores<D, false>(tmem + L::kTmDPt, 0u, v_kmaj, at(do_kmaj, st * kTile16));
            umma_commit(bar_s_full);
            if (t + 1 == itm.n) umma_commit(bar_v_free);  // the item's last dP^T has been issued
          }
          ++u;
        }
        if (!ok) bwd_timeout(a.status, abort_flag);
      } else {
        // ------------------------------------------------------------ gradient MMAs
        for (int k = 0, w; (w = pipe_item_index(k)) < n_items && ok; ++k) {
          const PipeItem itm = pipe_item<kSparse>(a, w);
          if (itm.n <= 0) continue;
          const int ks = u & 1;
          for (int t = 0; t < itm.n; ++t, ++T) {
            const int st = T % L::kQStages;
            const int db = T % L::kDsBufs;
            if (!mbar_wait(bar_p_full, T & 1, a.timeout_ns) || *abort_flag) {
              ok = false;
              break;
            }
            // the previous item's dK / dV must have left tensor memory before they restart
            if (t == 0 && u > 0 && (!mbar_wait(bar_acc_free, (u - 1) & 1, a.timeout_ns) || *abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_acc_tmem_linear<D>(tmem + L::kTmDV, tmem + L::kTmPt, at(do_mn, st * kTile16), t == 0);
            umma_commit(bar_pt_free);  // P^T is no longer read
            issue_acc<D, false>(tmem + L::kTmDK, 0u, at(ds_kmaj, db * kDs16), at(q_mn, st * kTile16), t == 0);
            umma_commit(bar_q_empty + st);  // nor are Q and dO of this tile
            if (T > 0) {                    // the previous dQ tile must have left tensor memory
              if (!mbar_wait(bar_dq_empty, (T - 1) & 1, a.timeout_ns) || *abort_flag) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            issue_dq<D>(tmem + L::kTmDQ, at(ds_mn, db * kDs16), at(k_mn, ks * kTile16));
            umma_commit(bar_dq_full);
            umma_commit(bar_ds_free + db);
            if (t + 1 == itm.n) {
              umma_commit(bar_k_free + ks);  // this K slot may be refilled
              umma_commit(bar_dkv_done);     // dK and dV of this item are complete
            }
          }
          ++u;
        }
        if (!ok) {
          bwd_timeout(a.status, abort_flag);
          umma_commit(bar_dkv_done);
        }
      }
    }
  } else if (warp < 8) {
    regs_dec<kPipeRegsDrain>();
    // ---------------------------------------------------------------- dQ drain (thread = query)
    const uint32_t quarter = warp & 3;
    const uint32_t lane_field = (quarter * 32) << 16;
    const int rr_sub = lane >> 3, cc = lane & 7;  // read side: row 4k + rr_sub, chunk cc
    bool ok = true;
    PipeCursor<kSparse> cur;
    cur.start(a, n_items);
    for (int T = 0; cur.valid; ++T, cur.advance(a, n_items)) {
      const int q0 = cur.qtile() * 128 + quarter * 32;  // first query row of this warp
      // this warp's 4 KB turn-around buffer in the drained tile's dS buffer:
      // row = lane, 16-byte chunk c at (c ^ (row & 7))
      const uint32_t scratch = sbase + L::kOffDS + (T % L::kDsBufs) * L::kDsBytes + quarter * 4096;
      if (!warp_wait_b(bar_dq_full, T & 1, a.timeout_ns) || *abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t g[32];
        tmem_ld32(tmem + lane_field + L::kTmDQ + half * 32, g);
        tmem_ld_wait(g);
        if (half == 1) {  // the tile is out of tensor memory
          tc_fence_before();
          mbar_arrive_warp(bar_dq_empty);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(scratch + lane * 128 + ((c ^ (lane & 7)) << 4), g[4 * c], g[4 * c + 1], g[4 * c + 2],
                       g[4 * c + 3]);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int row = 4 * k + rr_sub;
          const float4 v = ld_shared_f4(scratch + row * 128 + ((cc ^ (row & 7)) << 4));
          if (q0 + row < cur.itm.s.lq)
            red_add_v4(a.dq_acc +
                           ((size_t)((long long)cur.itm.s.tb * a.Nq + cur.itm.s.tq + q0 + row) * a.H + cur.itm.h) * D +
                           half * 32 + cc * 4,
                       v.x, v.y, v.z, v.w);
        }
        __syncwarp();
      }
      mbar_arrive_warp(bar_ds_free + (T % L::kDsBufs));  // the scratch may be overwritten
      if (cur.t + 1 < cur.itm.n) continue;
      // ------------------------------------------------------------ dK / dV of this item
      // (the drain warps write them, so that the dS warps go straight on to the next
      // item's first query tile): one key row per thread, 32 columns at a time
      if (!warp_wait_b(bar_dkv_done, cur.u & 1, a.timeout_ns) || *abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int key = cur.itm.j * 128 + (int)(quarter * 32 + lane);
      const bool key_in = key < cur.itm.s.lk;
      const size_t row = ((size_t)((long long)cur.itm.s.tb * a.Nk + cur.itm.s.tk + key) * a.H + cur.itm.h) * (D / 8);
#pragma unroll 1
      for (int part = 0; part < 4; ++part) {  // dK columns 0-31, 32-63, then dV
        uint32_t g[32];
        tmem_ld32(tmem + lane_field + (part < 2 ? L::kTmDK : L::kTmDV) + (part & 1) * 32, g);
        tmem_ld_wait(g);
        if (part == 3) {  // dK and dV are out of tensor memory: the next item may restart them
          tc_fence_before();
          mbar_arrive_warp(bar_acc_free);
        }
        if (key_in) {
          const float mul = part < 2 ? a.scale : 1.f;
          uint4* dst = (part < 2 ? a.dk : a.dv) + row + (part & 1) * 4;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t* f = g + 8 * c;
            dst[c] = make_uint4(pack_bf16x2(__uint_as_float(f[0]) * mul, __uint_as_float(f[1]) * mul),
                                pack_bf16x2(__uint_as_float(f[2]) * mul, __uint_as_float(f[3]) * mul),
                                pack_bf16x2(__uint_as_float(f[4]) * mul, __uint_as_float(f[5]) * mul),
                                pack_bf16x2(__uint_as_float(f[6]) * mul, __uint_as_float(f[7]) * mul));
          }
        }
      }
    }
    if (!ok && lane == 0) bwd_timeout(a.status, abort_flag);
  } else {
    regs_inc<kPipeRegsDs>();
    // ---------------------------------------------------------------- dS warps (thread = key)
    const uint32_t quarter = warp & 3;
    const int grp = (warp - 8) >> 2;  // column group: queries [64 grp, 64 grp + 64) of each tile
    const int r = quarter * 32 + lane;
    const uint32_t lane_field = (quarter * 32) << 16;
    const int col = 64 * grp;
    bool ok = true;
    int T = 0;
    for (int k = 0, w; (w = pipe_item_index(k)) < n_items && ok; ++k) {
      const PipeItem itm = pipe_item<kSparse>(a, w);
      if (itm.n <= 0) {
        if (itm.s.lq < 0) {
          if (threadIdx.x == 256) atomicExch(a.status, kStatusBadArg);
        } else if (itm.n == 0) {
          store_zero_dkv<D>(a, itm.s, itm.j, itm.h, threadIdx.x - 256, 256);
        }
        continue;
      }
      const int key = itm.j * 128 + r;
      const bool key_ok = key < itm.s.lk && key_attended(a, itm.b, key);  // P not masked out
      const int qmin = a.causal ? key - (itm.s.lk - itm.s.lq + a.causal_delta) : -(1 << 30);
      const bool key_tail = a.key_mask != nullptr || itm.j * 128 + 128 > itm.s.lk;  // masked variant
      const int last_key_qmin = itm.j * 128 + 127 - (itm.s.lk - itm.s.lq + a.causal_delta);
      const int n_qt = (itm.s.lq + 127) >> 7;
      int qi = next_kept_q<kSparse>(a, itm.h, itm.j, itm.i_first, n_qt);  // query tile of step t
      for (int t = 0; t < itm.n; ++t, ++T, qi = next_kept_q<kSparse>(a, itm.h, itm.j, qi + 1, n_qt)) {
        const int st = T % L::kQStages;
        const int db = T % L::kDsBufs;
        const int q0 = (kSparse ? qi : itm.i_first + t) * 128;
        if (!warp_wait_b(bar_q_full + st, (T / L::kQStages) & 1, a.timeout_ns) ||
            !warp_wait_b(bar_s_full, T & 1, a.timeout_ns) || *abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv0[32], sv1[32], dp0[32], dp1[32];
        tmem_ld32(tmem + lane_field + L::kTmSt + col, sv0);
        tmem_ld32(tmem + lane_field + L::kTmSt + col + 32, sv1);
        tmem_ld32(tmem + lane_field + L::kTmDPt + col, dp0);
        tmem_ld32(tmem + lane_field + L::kTmDPt + col + 32, dp1);
        tmem_ld_wait(sv0);
        reg_pin(sv1);
        reg_pin(dp0);
        reg_pin(dp1);
        tc_fence_before();
        mbar_arrive_warp(bar_s_free);  // S^T / dP^T may be overwritten
        const uint32_t stat_u32 = sbase + L::kOffStat + st * 1024 + col * 4;
        const uint32_t ds_row = sbase + L::kOffDS + db * L::kDsBytes + grp * 16384 + r * 128;
        const int qs0 = q0 + col, qs1 = q0 + col + 32;
        // both 32-query blocks first: the waits for the P^T columns and the dS buffer
        // come as late as possible (storing the first block's P^T and dS while the
        // second is computed measured 1% slower)
        uint32_t pk0[16], dk0[16], pk1[16], dk1[16];
        if constexpr (kDrop) {
          const DropCtx dctx{a.drop_t, a.drop_scale, a.seed_lo, a.seed_hi, key, itm.h, itm.b};
          ds_block<32, true, true>(sv0, dp0, stat_u32, a.scale_log2, key_ok, qmin - qs0, pk0, dk0, &dctx, qs0);
          ds_block<32, true, true>(sv1, dp1, stat_u32 + 128, a.scale_log2, key_ok, qmin - qs1, pk1, dk1, &dctx,
                                   qs1);
        } else {
          if (key_tail || (a.causal && last_key_qmin > qs0))
            ds_block<32, true>(sv0, dp0, stat_u32, a.scale_log2, key_ok, qmin - qs0, pk0, dk0);
          else
            ds_block<32, false>(sv0, dp0, stat_u32, a.scale_log2, key_ok, qmin - qs0, pk0, dk0);
          if (key_tail || (a.causal && last_key_qmin > qs1))
            ds_block<32, true>(sv1, dp1, stat_u32 + 128, a.scale_log2, key_ok, qmin - qs1, pk1, dk1);
          else
            ds_block<32, false>(sv1, dp1, stat_u32 + 128, a.scale_log2, key_ok, qmin - qs1, pk1, dk1);
        }
        // P^T may be written once the previous tile's dV has read it
        if (T > 0 && (!warp_wait_b(bar_pt_free, (T - 1) & 1, a.timeout_ns) || *abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st16(tmem + lane_field + L::kTmPt + 32 * grp, pk0);
        tmem_st16(tmem + lane_field + L::kTmPt + 32 * grp + 16, pk1);
        if (!warp_wait_b(bar_ds_free + db, ((T / L::kDsBufs) & 1) ^ 1, a.timeout_ns) || *abort_flag) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          st_shared_v4(ds_row + ((c4 ^ (r & 7)) << 4), dk0[4 * c4], dk0[4 * c4 + 1], dk0[4 * c4 + 2], dk0[4 * c4 + 3]);
          st_shared_v4(ds_row + (((4 + c4) ^ (r & 7)) << 4), dk1[4 * c4], dk1[4 * c4 + 1], dk1[4 * c4 + 2],
                       dk1[4 * c4 + 3]);
        }
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive_warp(bar_p_full);
      }
      if (!ok) break;
      // dK and dV of this item are written by the drain warps
    }
    if (!ok && lane == 0) bwd_timeout(a.status, abort_flag);
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
  static PerDeviceOnce attr_once;
  if (!attr_once.run([] {
        auto set = [](const void* fn, int bytes) {
          return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
        };
        if constexpr (D == 64)
          return set((const void*)bwd_pipe_kernel<false, false>, PipeLayout::kSmemBytes) &&
                 set((const void*)bwd_pipe_kernel<true, false>, PipeLayout::kSmemBytes) &&
                 set((const void*)bwd_pipe_kernel<false, true>, PipeLayout::kSmemBytes);
        else
          return set((const void*)bwd_main_kernel<D, false, false>, L::kSmemBytes) &&
                 set((const void*)bwd_main_kernel<D, true, false>, L::kSmemBytes) &&
                 set((const void*)bwd_main_kernel<D, false, true>, L::kSmemBytes);
      }))
    return FA_ERR_CUDA;
  // A packed batch is one batch element of total rows for the tensor maps, the
  // preprocess and the convert kernels; the main kernels find each sequence's rows.
  const bool varlen = L0.cu_q != nullptr;
  const int mB = varlen ? 1 : L0.B;
  const int mNq = varlen ? L0.total_q : L0.Nq, mNk = varlen ? L0.total_k : L0.Nk;
  // 1. D rows and a zeroed dQ accumulator
  {
    const long long rows = (long long)mB * mNq * L0.H;
    const long long threads = rows * (D / 8);
    const int grid = (int)((threads + 255) / 256);
    prof_before(stream, kKBwdPre);
    bwd_preprocess_kernel<D><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(L0.o),
                                                         static_cast<const __nv_bfloat16*>(L0.dout), L0.delta,
                                                         L0.dq_acc, mB, L0.H, mNq);
    const cudaError_t err = cudaGetLastError();
    prof_after(stream, kKBwdPre);
    if (err != cudaSuccess) return FA_ERR_CUDA;
  }
  // 2. main kernel
  CUtensorMap tq, tk, tv, tdo, tdk, tdv;
  if (!encode_bshd_map(&tq, L0.q, mB, mNq, L0.H, D) || !encode_bshd_map(&tk, L0.k, mB, mNk, L0.H, D) ||
      !encode_bshd_map(&tv, L0.v, mB, mNk, L0.H, D) || !encode_bshd_map(&tdo, L0.dout, mB, mNq, L0.H, D) ||
      !encode_bshd_map(&tdk, L0.dk, mB, mNk, L0.H, D) || !encode_bshd_map(&tdv, L0.dv, mB, mNk, L0.H, D))
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
  a.dk = static_cast<uint4*>(L0.dk);
  a.dv = static_cast<uint4*>(L0.dv);
  a.cu_q = L0.cu_q;
  a.cu_k = L0.cu_k;
  a.total_q = L0.total_q;
  a.total_k = L0.total_k;
  a.stat_n = mNq;
  a.key_mask = L0.key_mask;
  a.km_words = (L0.Nk + 31) / 32;
  a.drop_t = L0.drop_t;
  a.drop_scale = L0.drop_t ? (float)(65536.0 / (65536.0 - (double)L0.drop_t)) : 1.f;
  a.seed_lo = (uint32_t)(L0.seed & 0xFFFFFFFFull);
  a.seed_hi = (uint32_t)(L0.seed >> 32);
  a.block_mask = L0.block_mask;
  a.nqb = (L0.Nq + 127) / 128;
  a.nkb = (L0.Nk + 127) / 128;
  a.causal_delta = L0.causal_delta;
  const long long grid = (long long)a.n_kv_tiles * L0.B * L0.H;
  if (grid > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  prof_before(stream, kKBwdMain);
  if constexpr (D == 64) {
    const int pgrid = (int)std::min<long long>(grid, (long long)num_sms());
    if (a.block_mask != nullptr)
      bwd_pipe_kernel<false, true><<<pgrid, kPipeThreads, PipeLayout::kSmemBytes, stream>>>(tq, tk, tv, tdo, a);
    else if (a.drop_t != 0u)
      bwd_pipe_kernel<true, false><<<pgrid, kPipeThreads, PipeLayout::kSmemBytes, stream>>>(tq, tk, tv, tdo, a);
    else
      bwd_pipe_kernel<false, false><<<pgrid, kPipeThreads, PipeLayout::kSmemBytes, stream>>>(tq, tk, tv, tdo, a);
  } else {
    if (a.block_mask != nullptr)
      bwd_main_kernel<D, false, true>
          <<<(unsigned)grid, kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, tdo, tdk, tdv, a);
    else if (a.drop_t != 0u)
      bwd_main_kernel<D, true, false>
          <<<(unsigned)grid, kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, tdo, tdk, tdv, a);
    else
      bwd_main_kernel<D, false, false>
          <<<(unsigned)grid, kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, tdo, tdk, tdv, a);
  }
  const cudaError_t err_main = cudaGetLastError();
  prof_after(stream, kKBwdMain);
  if (err_main != cudaSuccess) return FA_ERR_CUDA;
  // 3. dQ = scale * accumulator in bf16
  {
    const long long n8 = (long long)mB * mNq * L0.H * D / 8;
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
