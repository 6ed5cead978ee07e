// fwd_sm100.cu -- exact attention forward pass for B200 (sm_100a).
//
// What it computes ("FlashAttention saves IO, not N^2 work", sections 1-3; Flash
// Attention wiki note, "Online Softmax", "Tiling" and "Flash Attention V2 的改进"):
// for every (batch b, head h, query row i)
//     o_i   = sum_j softmax_j(scale * q_i . k_j) v_j
//     lse_i = ln sum_j exp(scale * q_i . k_j)
// visiting the keys one 128-row tile at a time with the running (m, l, u) row
// state, so the score and probability tiles only ever live in tensor memory.
//
// B200 design
//  * Work item = (b, h, pair of 128-row query tiles).  Persistent grid, one CTA
//    per SM; items are numbered heaviest (latest causal rows) first and handed out
//    in that order by a counter in the workspace: the producer warp takes the next
//    one whenever it starts an item and publishes it to the other roles through a
//    small ring in shared memory, so a CTA that drew light items simply takes more
//    (a static order left the busiest SM 10% above the mean at the GPT-2-medium
//    shape; sequences of different lengths leave some items empty).
//  * Warp roles (384 threads, three warpgroups):
//      warp 0      TMA producer: Q tiles, then K/V tiles through a ring of smem
//                  slots (mbarrier full/empty pairs).
//      warp 1      TMEM allocator and tcgen05.mma issuer (one thread).
//      warps 2-3   idle (they complete the first warpgroup, which hands most of
//                  its registers to the softmax warpgroups).
//      warps 4-7   softmax group for query tile 0, warps 8-11 for tile 1; thread
//                  = query row = TMEM lane.
//  * Tensor memory (512 columns), d = 128: S0 [0,128), S1 [128,256), O0 [256,384),
//    O1 [384,512); P (bf16) is written over the first 64 columns of its S tile
//    and fed to the P.V MMA directly from tensor memory.  The two query tiles
//    ping-pong: while one softmax group works on its scores the tensor core runs
//    the other tile's MMAs.
//  * d = 64 has room for separate P columns: S0, S1 [0,256), P0 [256,320),
//    P1 [320,384), O0 [384,448), O1 [448,512).  A softmax group copies its S tile
//    into registers and releases it at once, so the next Q K^T of the same query
//    tile runs while the group works; one thread issues the Q K^T MMAs (warp 1)
//    and another the P V MMAs (warp 2), each as soon as its operands are ready.
//  * Online softmax in the log2 domain (x = s * scale * log2 e).  The running
//    max is only moved when a tile raises it by more than 8 (a factor 256), so
//    the O rescale (a TMEM round trip) is rare; the result is unchanged because
//    numerator and denominator use the same reference.  The 1/l normalisation
//    happens once, in the epilogue.  Two row sums are kept: the sum of the
//    bf16-rounded probabilities (exactly the weights the P.V MMA used) divides
//    O, and the sum of the unrounded ones gives lse.
//  * Per score element the softmax issues few instructions: packed fp32x2 FMA
//    (scale and subtract), MUFU exp2, packed bf16 conversion and packed fp32x2
//    adds into the two row sums; the row max uses 3-input max.
//  * Causal (bottom-right aligned): KV tiles entirely above the diagonal are
//    never loaded or multiplied; only tiles that cross it are masked.
//  * Variable-length batches (packed [total, H, d] rows with cu_seqlens): an item
//    reads its sequence's offsets and lengths; the TMA maps see one long batch,
//    keys past the sequence's end are masked like the causal triangle, and a
//    query tile that ends inside its sequence is stored by TMA while the last,
//    partial tile of a sequence writes its own rows directly, so no store reaches
//    the next sequence.  Offsets that do not fit the buffers are recorded in the
//    status word and the sequence is skipped.
//  * Epilogue: O/l -> bf16 -> swizzled smem (the Q tile's slot) -> TMA store;
//    lse as coalesced fp32 stores.
#include "fa_internal.h"
#include "philox.cuh"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr int kThreads = 384;
// Register split: launched at 168 per thread (384 x 168 = 64512); the producer /
// MMA warpgroup drops to 80 and the two softmax warpgroups rise to 208:
// 128 x 80 + 256 x 208 = 63488.
constexpr uint32_t kRegsLow = 80, kRegsHigh = 208;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= 384 * 168, "register split exceeds the launch budget");
constexpr uint32_t kTmemCols = 512;
// tensor-memory column of the score tile / O accumulator of query tile t
__host__ __device__ constexpr uint32_t tm_s(int t) { return t * 128u; }
// separate P columns (d = 64): S is released as soon as the softmax has read it
template <int D>
__host__ __device__ constexpr bool sep_p() {
  return D == 64;
}
template <int D>
__host__ __device__ constexpr uint32_t tm_p(int t) {
  return sep_p<D>() ? 256u + 64u * t : tm_s(t);
}
template <int D>
__host__ __device__ constexpr uint32_t tm_o(int t) {
  return sep_p<D>() ? 384u + 64u * t : 256u + t * 128u;
}
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Polls before a sleeping wait: the MMA issuer (one thread, on the tensor core's
// critical path) and the softmax warps waiting for their scores.
#ifndef FA_FWD_MMA_SPINS
#define FA_FWD_MMA_SPINS 0
#endif
#ifndef FA_FWD_SOFTMAX_SPINS
#define FA_FWD_SOFTMAX_SPINS 0
#endif
constexpr int kMmaSpins = FA_FWD_MMA_SPINS;
constexpr int kSoftmaxSpins = FA_FWD_SOFTMAX_SPINS;
// Every kExpFmaEvery-th group of four probabilities computes one pair of its
// exponentials on the FMA pipes (exp2_fma2) instead of the MUFU unit: an eighth of
// them at d = 64, a sixteenth at d = 128.  Measured on B200 against other splits
// (at d = 64 a quarter was 5% slower, a sixteenth within 1%; at d = 128, with the
// P V in two halves, a sixteenth 0.7% faster than an eighth and a quarter 3%
// slower).
#ifndef FA_FWD_EXP_FMA_EVERY_128
#define FA_FWD_EXP_FMA_EVERY_128 8
#endif
#ifndef FA_FWD_EXP_FMA_EVERY_64
#define FA_FWD_EXP_FMA_EVERY_64 4
#endif
template <int D>
__host__ __device__ constexpr int exp_fma_every() {
  return D == 64 ? FA_FWD_EXP_FMA_EVERY_64 : FA_FWD_EXP_FMA_EVERY_128;
}

template <int D>
struct FwdLayout {
  static constexpr int kTileBytes = 128 * D * 2;   // one 128-row bf16 tile of Q, K or V
  static constexpr int kBoxes = D / 64;            // 64-column (128-byte) TMA boxes per tile
  static constexpr int kBoxBytes = 128 * 128;      // 16 KB
  static constexpr int kStages = (D == 64) ? 8 : 4;
  static constexpr int kOffQ = 0;                  // Q tile 0, Q tile 1
  static constexpr int kOffRing = 2 * kTileBytes;
  // d = 64 has room for an output staging buffer of its own (two tiles), so the Q
  // pair is released as soon as the item's last Q K^T MMA has read it and the next
  // item's Q load overlaps this item's last steps and epilogue; d = 128 stages its
  // output through the Q tiles and releases them after the epilogue.
  static constexpr bool kEarlyQ = (D == 64);
  static constexpr int kOffStage = kOffRing + kStages * kTileBytes;
  static constexpr int kOffBar = kOffStage + (kEarlyQ ? 2 * kTileBytes : 0);
  // barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2], epi[2],
  // s_free[2], p_free[2], stage_free[2], item_full[R], item_empty[R]
  static constexpr int kItemRing = 4;  // items the producer may publish ahead of the other roles
  static constexpr int kNumBars = 2 + 2 * kStages + 14 + 2 * kItemRing;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffItems = kOffMisc + 64;  // the item ring: int per slot
  static constexpr int kSmemBytes = kOffItems + 4 * kItemRing + 1024;  // + alignment slack
};

struct FwdArgs {
  float* lse;
  int* status;
  __nv_bfloat16* o;  // for the direct stores of partial variable-length tiles
  const int32_t* cu_q;  // variable-length batch: [B + 1] row offsets (null for a dense batch)
  const int32_t* cu_k;
  int total_q, total_k;
  int B, H, Nq, Nk;  // variable length: Nq, Nk are the maximum sequence lengths
  int causal;
  float scale_log2;
  int n_pairs;
  int n_items;
  // items are handed out in order (heaviest first) by a counter in the workspace;
  // the last CTA to finish resets it and the exit count for the next call
  unsigned int* item_ctr;
  unsigned int* done_ctr;
  unsigned long long timeout_ns;
  // key-padding mask (null: none): [B, km_words] bits, bit j % 32 of word j / 32
  // set when key j of the batch element takes part
  const uint32_t* key_mask;
  int km_words;
  // dropout (drop_t = 0: none): a probability is kept when its 16-bit draw is at
  // least drop_t and then scaled by drop_scale (philox.cuh gives the draws)
  uint32_t drop_t;
  float drop_scale;
  uint32_t seed_lo, seed_hi;
  // block-sparse mask (null: dense): [H, nqb, nkb] bytes over (128-row query
  // tile, 128-key KV tile); 0 skips the block
  const uint8_t* block_mask;
  int nqb, nkb;
  // causal: query i sees key j iff j <= i + (lk - lq) + causal_delta (0 except for a
  // key shard, whose keys start later in the sequence)
  int causal_delta;
};

// KV tile j takes part for 128-row query tile qtile of head h (always in the dense
// instantiation).
template <bool kSparse>
__device__ __forceinline__ bool block_kept(const FwdArgs& a, int h, int qtile, int j) {
  if constexpr (!kSparse) return true;
  return __ldg(a.block_mask + ((size_t)h * a.nqb + qtile) * a.nkb + j) != 0;
}

// The 128 mask bits of KV tile j of batch element b (all set without a mask;
// words past the row are 0, their keys are past the end anyway).
__device__ __forceinline__ void tile_mask_words(const FwdArgs& a, int b, int j, uint32_t (&w)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = ~0u;
  if (a.key_mask == nullptr) return;
  const uint32_t* row = a.key_mask + (size_t)b * a.km_words;
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = (j * 4 + i < a.km_words) ? __ldg(row + j * 4 + i) : 0u;
}


__device__ __forceinline__ void item_coords(const FwdArgs& a, int w, int& b, int& h, int& pair) {
  const int bh_count = a.B * a.H;
  const int pr = w / bh_count;
  const int bh = w - pr * bh_count;
  pair = a.causal ? (a.n_pairs - 1 - pr) : pr;
  b = bh / a.H;
  h = bh - b * a.H;
}

// The rows of sequence b: query rows qoff .. qoff + lq - 1 and key rows
// koff .. koff + lk - 1 of the batch coordinate bc.  A dense batch has lq = Nq,
// lk = Nk at offset 0 of batch b; a variable-length batch reads cu_seqlens
// (lq = -1 marks a sequence whose offsets do not fit the buffers).
struct SeqView {
  int lq, lk, qoff, koff, bc;
};
__device__ __forceinline__ SeqView seq_view(const FwdArgs& a, int b) {
  SeqView v;
  if (a.cu_q == nullptr) {
    v.lq = a.Nq;
    v.lk = a.Nk;
    v.qoff = 0;
    v.koff = 0;
    v.bc = b;
    return v;
  }
  v.qoff = a.cu_q[b];
  v.koff = a.cu_k[b];
  const int q1 = a.cu_q[b + 1], k1 = a.cu_k[b + 1];
  v.bc = 0;
  // no expression below can wrap: ends are compared with starts before they are
  // subtracted, and the fit is checked against total - start (both non-negative)
  if (v.qoff < 0 || v.koff < 0 || q1 < v.qoff || k1 < v.koff) {
    v.lq = -1;
    v.lk = 0;
    return v;
  }
  v.lq = min(q1 - v.qoff, a.Nq);
  v.lk = min(k1 - v.koff, a.Nk);
  if (v.lq > a.total_q - v.qoff || v.lk > a.total_k - v.koff) v.lq = -1;
  return v;
}

// Number of KV tiles query tile starting at row0 needs; -1 when the tile is empty.
__device__ __forceinline__ int tile_kv_count(const FwdArgs& a, const SeqView& v, int row0) {
  if (row0 >= v.lq) return -1;
  if (!a.causal) return (v.lk + 127) >> 7;
  const int last = min(row0 + 127, v.lq - 1);
  long long kend = (long long)last + 1 + v.lk - v.lq + a.causal_delta;
  if (kend <= 0) return 0;
  if (kend > v.lk) kend = v.lk;
  return (int)((kend + 127) >> 7);
}

__device__ __forceinline__ void record_timeout(int* status, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicCAS(status, 0, kStatusTimeout);
}

// Warp-uniform bounded wait: lane 0 waits, the verdict is broadcast.
template <int kSpins = 0>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, unsigned long long timeout_ns) {
  bool ok = true;
  if (lane_id() == 0) ok = mbar_wait_spin<kSpins>(bar, parity, timeout_ns);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// S = Q K^T for one 128x128 tile: K-major operands, 16-wide k-steps of 32 bytes
// inside each 128-byte swizzle row, 64-column boxes 16 KB apart.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, SDesc q, SDesc k) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * 1024 + (kk & 3) * 2;  // 16-byte units
    umma_ss(d_tmem, sdesc_at(q, off), sdesc_at(k, off), idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V: P bf16 in tensor memory (8 columns per 16 keys), V MN-major in smem
// (16 keys = 2048 bytes per k-step).
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, SDesc v, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    umma_ts(o_tmem, p_tmem + kk * 8, sdesc_at(v, kk * 128), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// One half of issue_pv: keys 64 half .. 64 half + 63.
template <int D>
__device__ __forceinline__ void issue_pv_half(uint32_t o_tmem, uint32_t p_tmem, SDesc v, bool accumulate, int half) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
#pragma unroll
  for (int k4 = 0; k4 < 4; ++k4) {
    const int kk = 4 * half + k4;
    umma_ts(o_tmem, p_tmem + kk * 8, sdesc_at(v, kk * 128), idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// kDrop: dropout on P; kSparse: block-sparse attention (separate instantiations,
// so the plain kernel is unchanged)
template <int D, bool kDrop, bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const FwdArgs a) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* bar_q_full = bars + 0;
  uint64_t* bar_q_empty = bars + 1;
  uint64_t* bar_kv_full = bars + 2;
  uint64_t* bar_kv_empty = bars + 2 + L::kStages;
  uint64_t* bar_s_full = bars + 2 + 2 * L::kStages;
  uint64_t* bar_p_full = bar_s_full + 2;
  uint64_t* bar_o_done = bar_s_full + 4;
  uint64_t* bar_epi = bar_s_full + 6;
  uint64_t* bar_s_free = bar_s_full + 8;  // separate P: the softmax group has read S
  // P over S (d = 128), which has no use for s_free: the P of the tile's first 64
  // keys is in tensor memory (one arrival per softmax warp), so that their P V
  // runs while the softmax computes the other half
  uint64_t* bar_p_half = bar_s_full + 8;
  uint64_t* bar_p_free = bar_s_full + 10;  // separate P: the P V MMA has read P
  uint64_t* bar_stage_free = bar_s_full + 12;  // early Q release: the output staging buffer is free
  uint64_t* bar_item_full = bar_s_full + 14;                // [kItemRing]: the producer published an item
  uint64_t* bar_item_empty = bar_item_full + L::kItemRing;  // [kItemRing]: every other role has read it
  volatile int* item_ring = reinterpret_cast<volatile int*>(smem + L::kOffItems);
  // roles that read the item ring: the MMA issuer warp(s) and the eight softmax warps
  constexpr uint32_t kItemReaders = (sep_p<D>() ? 2 : 1) + 8;
  constexpr bool kSepP = sep_p<D>();
  static_assert(L::kEarlyQ == kSepP, "the separate-P issuers are the ones that release Q early");
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 8);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const uint32_t smem_base = smem_u32(smem);

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, L::kEarlyQ ? 1 : 2);  // the Q K^T issuer, or both epilogues
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar_kv_full + s, 1);
      mbar_init(bar_kv_empty + s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full + t, 1);
      mbar_init(bar_p_full + t, 4);  // one arrival per softmax warp
      mbar_init(bar_o_done + t, 1);
      mbar_init(bar_epi + t, 4);
      mbar_init(bar_s_free + t, 4);  // one arrival per softmax warp
      mbar_init(bar_p_free + t, 1);
      mbar_init(bar_stage_free + t, 1);
    }
    for (int r2 = 0; r2 < L::kItemRing; ++r2) {
      mbar_init(bar_item_full + r2, 1);
      mbar_init(bar_item_empty + r2, kItemReaders);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_slot;

  if (warp < 4) {
   regs_dec<kRegsLow>();
   if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t item_iter = 0, g = 0;
      for (int n = 0; !*abort_flag; ++n) {
        // take the next item and publish it to the other roles (-1: none left)
        const int slot_i = n % L::kItemRing;
        if (!mbar_wait(bar_item_empty + slot_i, ((n / L::kItemRing) & 1) ^ 1, a.timeout_ns)) {
          record_timeout(a.status, abort_flag);
          break;
        }
        const unsigned int taken = atomicAdd(a.item_ctr, 1u);
        const int w = taken < (unsigned)a.n_items ? (int)taken : -1;
        item_ring[slot_i] = w;
        mbar_arrive(bar_item_full + slot_i);
        if (w < 0) break;
        int b, h, pair;
        item_coords(a, w, b, h, pair);
        const SeqView sv = seq_view(a, b);
        const int row0 = pair * 256;
        const int n0 = tile_kv_count(a, sv, row0), n1 = tile_kv_count(a, sv, row0 + 128);
        const int nkv = max(n0, n1);
        if (n0 < 0) continue;  // no query row of this item exists: every role skips it
        if (!mbar_wait(bar_q_empty, (item_iter++ & 1) ^ 1, a.timeout_ns)) {
          record_timeout(a.status, abort_flag);
          break;
        }
        mbar_arrive_expect_tx(bar_q_full, 2 * L::kTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int bx = 0; bx < L::kBoxes; ++bx)
            tma_load_4d(smem + L::kOffQ + t * L::kTileBytes + bx * L::kBoxBytes, &tmQ, bar_q_full, bx * 64, h,
                        sv.qoff + row0 + t * 128, sv.bc);
        for (int j = 0; j < nkv; ++j) {
          // KV tiles that neither query tile keeps are never loaded
          if (!((j < n0 && block_kept<kSparse>(a, h, 2 * pair, j)) || (j < n1 && block_kept<kSparse>(a, h, 2 * pair + 1, j))))
            continue;
          for (int kv = 0; kv < 2; ++kv, ++g) {
            const uint32_t slot = g % L::kStages, phase = (g / L::kStages) & 1;
            if (!mbar_wait(bar_kv_empty + slot, phase ^ 1, a.timeout_ns)) {
              record_timeout(a.status, abort_flag);
              j = nkv;
              break;
            }
            mbar_arrive_expect_tx(bar_kv_full + slot, L::kTileBytes);
            uint8_t* dst = smem + L::kOffRing + slot * L::kTileBytes;
            for (int bx = 0; bx < L::kBoxes; ++bx)
              tma_load_4d(dst + bx * L::kBoxBytes, kv == 0 ? &tmK : &tmV, bar_kv_full + slot, bx * 64, h,
                          sv.koff + j * 128, sv.bc);
          }
        }
      }
    }
  } else if (kSepP && (warp == 1 || warp == 2)) {
    // ------------------------------------------------------------------ MMA issuers (separate P)
    if (lane == 0) {
      const SDesc q_desc[2] = {sdesc_make(smem_base + L::kOffQ, 16, 1024),
                               sdesc_make(smem_base + L::kOffQ + L::kTileBytes, 16, 1024)};
      const SDesc ring_k = sdesc_make(smem_base + L::kOffRing, 16, 1024);     // K tiles, K-major
      const SDesc ring_v = sdesc_make(smem_base + L::kOffRing, 16384, 1024);  // V tiles, MN-major
      constexpr uint32_t kSlot16 = L::kTileBytes / 16;
      bool ok = true;
      auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) {
        if (!ok) return false;
        if (!mbar_wait_spin<kMmaSpins>(bar, parity, a.timeout_ns) || *abort_flag) {
          record_timeout(a.status, abort_flag);
          ok = false;
        }
        return ok;
      };
      // the next item from the producer's ring
      auto read_item = [&](int n, int& w) {
        const int slot_i = n % L::kItemRing;
        if (!wait_or_abort(bar_item_full + slot_i, (n / L::kItemRing) & 1)) return false;
        w = item_ring[slot_i];
        mbar_arrive(bar_item_empty + slot_i);
        return true;
      };
      // ring slots alternate K, V per KV step: K of step j at g, V at g + 1
      uint32_t item_iter = 0, g = 0;
      uint32_t cnt[2] = {0, 0};  // Q K^T (warp 1) or P V (warp 2) MMAs issued per query tile
      for (int n = 0; ok; ++n) {
        int w = -1;
        if (!read_item(n, w)) break;
        if (w < 0) break;
        int b, h, pair;
        item_coords(a, w, b, h, pair);
        const SeqView sv = seq_view(a, b);
        const int row0 = pair * 256;
        const int nt[2] = {tile_kv_count(a, sv, row0), tile_kv_count(a, sv, row0 + 128)};
        const int nkv = max(nt[0], nt[1]);
        if (nt[0] < 0) continue;  // no query row of this item exists: every role skips it
        const uint32_t it_q = item_iter++;  // items processed: q_full phases
        if (warp == 1) {
          // S_t = Q_t K_j^T once the group has read its previous S tile
          if (!wait_or_abort(bar_q_full, it_q & 1)) break;
          tc_fence_after();
          for (int j = 0; j < nkv && ok; ++j) {
            const bool kp[2] = {j < nt[0] && block_kept<kSparse>(a, h, 2 * pair, j),
                                j < nt[1] && block_kept<kSparse>(a, h, 2 * pair + 1, j)};
            if (!kp[0] && !kp[1]) continue;  // not in the item's KV stream
            const uint32_t slot_k = g % L::kStages;
            if (!wait_or_abort(bar_kv_full + slot_k, (g / L::kStages) & 1)) break;
            tc_fence_after();
            const SDesc k_desc = SDesc{ring_k.lo + slot_k * kSlot16, ring_k.hi};
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (kp[t]) {
                if (cnt[t] > 0 && !wait_or_abort(bar_s_free + t, (cnt[t] - 1) & 1)) break;
                tc_fence_after();
                issue_qk<D>(tmem_base + tm_s(t), q_desc[t], k_desc);
                umma_commit(bar_s_full + t);
                ++cnt[t];
              }
            }
            if (!ok) break;
            umma_commit(bar_kv_empty + slot_k);
            g += 2;
          }
          if (ok) umma_commit(bar_q_empty);  // arrives once every Q K^T of the item has read Q
        } else {
          // O_t += P_t V_j once the group has written P.  (No wait for the item's Q
          // here: the Q K^T issuer may already have released it and the producer
          // loaded the next item's, so its phase could have moved twice.)
          bool started[2] = {false, false};  // the tile's O holds a product of this item
          for (int j = 0; j < nkv && ok; ++j) {
            const bool kp[2] = {j < nt[0] && block_kept<kSparse>(a, h, 2 * pair, j),
                                j < nt[1] && block_kept<kSparse>(a, h, 2 * pair + 1, j)};
            if (!kp[0] && !kp[1]) continue;  // not in the item's KV stream
            const uint32_t slot_v = (g + 1) % L::kStages;
            if (!wait_or_abort(bar_kv_full + slot_v, ((g + 1) / L::kStages) & 1)) break;
            tc_fence_after();
            const SDesc v_desc = SDesc{ring_v.lo + slot_v * kSlot16, ring_v.hi};
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (kp[t]) {
                if (!wait_or_abort(bar_p_full + t, cnt[t] & 1)) break;
                tc_fence_after();
                issue_pv<D>(tmem_base + tm_o<D>(t), tmem_base + tm_p<D>(t), v_desc, started[t]);
                started[t] = true;
                umma_commit(bar_p_free + t);
                ++cnt[t];
              }
            }
            if (!ok) break;
            umma_commit(bar_kv_empty + slot_v);
            g += 2;
          }
          if (!ok) break;
          // both tiles' O are released together: releasing each right after its own
          // last P V measured 2% slower (its epilogue then competes with the other
          // tile's last step)
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if (nt[t] >= 0) umma_commit(bar_o_done + t);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t item_iter = 0, g = 0;
      uint32_t s_cnt[2] = {0, 0}, p_cnt[2] = {0, 0};
      const SDesc q_desc[2] = {sdesc_make(smem_base + L::kOffQ, 16, 1024),
                               sdesc_make(smem_base + L::kOffQ + L::kTileBytes, 16, 1024)};
      const SDesc ring_k = sdesc_make(smem_base + L::kOffRing, 16, 1024);      // K tiles, K-major
      const SDesc ring_v = sdesc_make(smem_base + L::kOffRing, 16384, 1024);   // V tiles, MN-major
      constexpr uint32_t kSlot16 = L::kTileBytes / 16;
      bool ok = true;
      auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) {
        if (!ok) return false;
        if (!mbar_wait_spin<kMmaSpins>(bar, parity, a.timeout_ns) || *abort_flag) {
          record_timeout(a.status, abort_flag);
          ok = false;
        }
        return ok;
      };
      // the next item from the producer's ring
      auto read_item = [&](int n, int& w) {
        const int slot_i = n % L::kItemRing;
        if (!wait_or_abort(bar_item_full + slot_i, (n / L::kItemRing) & 1)) return false;
        w = item_ring[slot_i];
        mbar_arrive(bar_item_empty + slot_i);
        return true;
      };
      for (int n = 0; ok; ++n) {
        int w = -1;
        if (!read_item(n, w)) break;
        if (w < 0) break;
        int b, h, pair;
        item_coords(a, w, b, h, pair);
        const SeqView sv = seq_view(a, b);
        const int row0 = pair * 256;
        const int nt[2] = {tile_kv_count(a, sv, row0), tile_kv_count(a, sv, row0 + 128)};
        const int nkv = max(nt[0], nt[1]);
        if (nt[0] < 0) continue;  // no query row of this item exists: every role skips it
        const uint32_t it_q = item_iter++;  // items processed: q_full phases
        if (!wait_or_abort(bar_q_full, it_q & 1)) break;
        tc_fence_after();
        if constexpr (kSparse) {
          // The item's KV stream: the tiles that at least one query tile keeps, in
          // order.  A tile's next scores are issued right after its P V (S and P
          // share columns; tcgen05 operations run in issue order).
          auto kept_t = [&](int t, int j) { return j < nt[t] && block_kept<kSparse>(a, h, 2 * pair + t, j); };
          auto next_in_stream = [&](int j) {
            for (int x = j + 1; x < nkv; ++x)
              if (kept_t(0, x) || kept_t(1, x)) return x;
            return nkv;
          };
          // first KV tile of the stream: first scores of the tiles that keep it
          int j = next_in_stream(-1);
          uint32_t slot_k = 0;
          if (j < nkv) {
            slot_k = g % L::kStages;
            if (!wait_or_abort(bar_kv_full + slot_k, (g / L::kStages) & 1)) break;
            tc_fence_after();
            ++g;
            const SDesc k_desc = SDesc{ring_k.lo + slot_k * kSlot16, ring_k.hi};
  #pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (kept_t(t, j)) {
                issue_qk<D>(tmem_base + tm_s(t), q_desc[t], k_desc);
                umma_commit(bar_s_full + t);
              }
            }
            umma_commit(bar_kv_empty + slot_k);
          }
          bool started[2] = {false, false};  // the tile's O holds a product of this item
          while (j < nkv && ok) {
            const int jn = next_in_stream(j);
            const uint32_t slot_v = g % L::kStages;
            if (!wait_or_abort(bar_kv_full + slot_v, (g / L::kStages) & 1)) break;
            tc_fence_after();
            ++g;
            const SDesc v_desc = SDesc{ring_v.lo + slot_v * kSlot16, ring_v.hi};
            const bool more = jn < nkv;
            SDesc k_desc = ring_k;
  #pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (kept_t(t, j)) {
                if (!wait_or_abort(bar_p_half + t, p_cnt[t] & 1)) break;
                tc_fence_after();
                issue_pv_half<D>(tmem_base + tm_o<D>(t), tmem_base + tm_s(t), v_desc, started[t], 0);
                if (!wait_or_abort(bar_p_full + t, p_cnt[t] & 1)) break;
                tc_fence_after();
                ++p_cnt[t];
                issue_pv_half<D>(tmem_base + tm_o<D>(t), tmem_base + tm_s(t), v_desc, true, 1);
                started[t] = true;
              }
              if (t == 0 && more) {
                slot_k = g % L::kStages;
                if (!wait_or_abort(bar_kv_full + slot_k, (g / L::kStages) & 1)) break;
                tc_fence_after();
                ++g;
                k_desc = SDesc{ring_k.lo + slot_k * kSlot16, ring_k.hi};
              }
              if (more && kept_t(t, jn)) {
                issue_qk<D>(tmem_base + tm_s(t), q_desc[t], k_desc);
                umma_commit(bar_s_full + t);
              }
            }
            if (!ok) break;
            umma_commit(bar_kv_empty + slot_v);
            if (more) umma_commit(bar_kv_empty + slot_k);
            j = jn;
          }
        } else {
          // K_0 : first scores of both tiles
          uint32_t slot_k = 0;
          if (nkv > 0) {
            slot_k = g % L::kStages;
            if (!wait_or_abort(bar_kv_full + slot_k, (g / L::kStages) & 1)) break;
            tc_fence_after();
            ++g;
            const SDesc k_desc = SDesc{ring_k.lo + slot_k * kSlot16, ring_k.hi};
  #pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (nt[t] > 0) {
                issue_qk<D>(tmem_base + tm_s(t), q_desc[t], k_desc);
                umma_commit(bar_s_full + t);
              }
            }
            umma_commit(bar_kv_empty + slot_k);
          }
          for (int j = 0; j < nkv && ok; ++j) {
            const uint32_t slot_v = g % L::kStages;
            if (!wait_or_abort(bar_kv_full + slot_v, (g / L::kStages) & 1)) break;
            tc_fence_after();
            ++g;
            const SDesc v_desc = SDesc{ring_v.lo + slot_v * kSlot16, ring_v.hi};
            const bool more = (j + 1 < nkv);
            SDesc k_desc = ring_k;
  #pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (j < nt[t]) {
                // the first 64 keys' P V as soon as their P is written
                if (!wait_or_abort(bar_p_half + t, p_cnt[t] & 1)) break;
                tc_fence_after();
                issue_pv_half<D>(tmem_base + tm_o<D>(t), tmem_base + tm_s(t), v_desc, j > 0, 0);
                if (!wait_or_abort(bar_p_full + t, p_cnt[t] & 1)) break;
                tc_fence_after();
                ++p_cnt[t];
                issue_pv_half<D>(tmem_base + tm_o<D>(t), tmem_base + tm_s(t), v_desc, true, 1);
              }
              if (t == 0 && more) {
                slot_k = g % L::kStages;
                if (!wait_or_abort(bar_kv_full + slot_k, (g / L::kStages) & 1)) break;
                tc_fence_after();
                ++g;
                k_desc = SDesc{ring_k.lo + slot_k * kSlot16, ring_k.hi};
              }
              if (more && j + 1 < nt[t]) {
                issue_qk<D>(tmem_base + tm_s(t), q_desc[t], k_desc);
                umma_commit(bar_s_full + t);
              }
            }
            if (!ok) break;
            umma_commit(bar_kv_empty + slot_v);
            if (more) umma_commit(bar_kv_empty + slot_k);
          }
        }
        if (!ok) break;
        // one completion per present tile and item: all of this tile's MMAs are done
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (nt[t] >= 0) umma_commit(bar_o_done + t);
        (void)s_cnt;
      }
    }
   }
  } else {
    regs_inc<kRegsHigh>();
    // ------------------------------------------------------------------ softmax groups
    const int t = (warp - 4) >> 2;               // query tile of this group
    const uint32_t quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;           // row within the tile
    const uint32_t lane_field = (quarter * 32) << 16;
    const uint32_t tS = tmem_base + lane_field + tm_s(t);
    const uint32_t tO = tmem_base + lane_field + tm_o<D>(t);
    const uint32_t tP = tmem_base + lane_field + tm_p<D>(t);
    const int tid_in_group = threadIdx.x - 128 - t * 128;
    uint32_t s_cnt = 0, tile_iter = 0;  // tile_iter counts items in which this tile is present
    uint32_t items_done = 0;            // items with a query row (the producer's q phases)
    // where the epilogue stages this tile's output for its TMA store
    uint8_t* o_stage = smem + (L::kEarlyQ ? L::kOffStage : L::kOffQ) + t * L::kTileBytes;
    const uint32_t o_stage_u32 = smem_u32(o_stage);

    for (int n = 0;; ++n) {
      int w = -1;
      {
        // the next item from the producer's ring (every lane gets the index)
        const int slot_i = n % L::kItemRing;
        if (!warp_wait(bar_item_full + slot_i, (n / L::kItemRing) & 1, a.timeout_ns)) {
          if (lane == 0) record_timeout(a.status, abort_flag);
          break;
        }
        w = item_ring[slot_i];
        mbar_arrive_warp(bar_item_empty + slot_i);
      }
      if (w < 0) break;
      if (*abort_flag) break;
      int b, h, pair;
      item_coords(a, w, b, h, pair);
      const SeqView sv = seq_view(a, b);
      if (sv.lq < 0 && pair == 0 && t == 0 && tid_in_group == 0) atomicExch(a.status, kStatusBadArg);
      const int row0 = pair * 256 + t * 128;
      const int nkv = tile_kv_count(a, sv, row0);
      // No query row of this item exists: every role skips it (an arrival here
      // could complete the producer's q_empty phase before its first wait).
      if (tile_kv_count(a, sv, pair * 256) < 0) continue;
      const uint32_t it_q = items_done++;
      if (nkv < 0) {
        // This query tile lies past the sequence: nothing to compute or store.
        if constexpr (L::kEarlyQ) continue;  // the Q K^T issuer releases the Q pair
        // Its release of the Q pair waits for this item's Q load, so that it can never
        // count toward the previous item's release (the other group may still be
        // staging that item's output in its Q tile).
        if (!warp_wait(bar_q_full, it_q & 1, a.timeout_ns) || *abort_flag) {
          if (lane == 0) record_timeout(a.status, abort_flag);
          break;
        }
        if (tid_in_group == 0) mbar_arrive(bar_q_empty);
        __syncwarp();
        continue;
      }
      const int row = row0 + r;
      // visible keys of this row: [0, lim)
      const int lk = sv.lk;  // only the key count stays live through the KV loop
      int lim = lk;
      const int cdelta = a.causal_delta;
      if (a.causal) lim = max(0, min(lk, row + 1 + lk - sv.lq + cdelta));
      const int group_first_lim = a.causal ? (row0 + 1 + lk - sv.lq + cdelta) : lk;  // smallest lim in the tile

      float m2 = -INFINITY;  // running reference max (log2 domain)
      float l = 0.f;         // running sum of the bf16-rounded probabilities (normalises O)
      float le = 0.f;        // running sum of the unrounded probabilities (gives lse)
      bool ok = true;
      int kept_n = 0;  // KV tiles of this item that this query tile has processed
      for (int j = 0; j < nkv; ++j) {
        if (!block_kept<kSparse>(a, h, 2 * pair + t, j)) continue;  // a skipped block: no scores were issued
        // Dropout: the keep bits of this row's 128 keys of KV tile j (bit c of word
        // c / 32 for key 128 j + c), drawn before the scores arrive (they depend on
        // nothing else).  One Philox call covers 4 rows x 2 keys, and rows 4i .. 4i+3
        // sit on four neighbouring lanes: each lane makes a quarter of the calls of
        // its quad and the four words of every call are handed round by shuffles.
        uint32_t keepw[4] = {~0u, ~0u, ~0u, ~0u};
        if constexpr (kDrop) {
          const uint32_t qd = lane & 3u;
          const uint32_t quad = lane & ~3u;
#pragma unroll
          for (int i = 0; i < 4; ++i) keepw[i] = 0u;
#pragma unroll 2
          for (int m = 0; m < 16; ++m) {  // key pairs 4m .. 4m + 3 of the tile: keys 8m .. 8m + 7
            const uint32_t kb = (uint32_t)j * 64u + 4u * m + qd;
            const uint4 w = philox4x32_10(make_uint4(kb, (uint32_t)row >> 2, (uint32_t)h, (uint32_t)b), a.seed_lo,
                                          a.seed_hi);
            uint32_t bits = 0u;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // lane s hands out the word of row (s - k) & 3; lane qd receives from lane
              // (qd + k) & 3 the word of its own row in that lane's call
              const uint32_t give = (qd - k) & 3u;
              const uint32_t v = give == 0 ? w.x : (give == 1 ? w.y : (give == 2 ? w.z : w.w));
              const uint32_t src = (qd + k) & 3u;
              const uint32_t got = __shfl_sync(0xffffffffu, v, (int)(quad | src));
              const uint32_t keep2 = ((got & 0xFFFFu) >= a.drop_t ? 1u : 0u) | ((got >> 16) >= a.drop_t ? 2u : 0u);
              bits |= keep2 << (2 * src);
            }
            keepw[m >> 2] |= bits << (8 * (m & 3));
          }
        }
        if (!warp_wait<kSoftmaxSpins>(bar_s_full + t, s_cnt & 1, a.timeout_ns) || *abort_flag) {
          if (lane == 0) record_timeout(a.status, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[4][32];
#pragma unroll
        for (int i = 0; i < 4; ++i) tmem_ld32(tS + i * 32, s[i]);
        tmem_ld_wait(s[0]);
        reg_pin(s[1]);
        reg_pin(s[2]);
        reg_pin(s[3]);
        if constexpr (kSepP) {  // the next Q K^T of this tile may overwrite S
          tc_fence_before();
          mbar_arrive_warp(bar_s_free + t);
        }

        // mask (only tiles that cross the diagonal or the key tail, or every tile
        // under a key-padding mask)
        const int kbase = j * 128;
        if (a.key_mask != nullptr || kbase + 128 > min(group_first_lim, lk) || kbase + 128 > lk) {
          uint32_t kmw[4];
          tile_mask_words(a, b, j, kmw);
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (kbase + i * 32 + c >= lim || !((kmw[i] >> c) & 1u)) s[i][c] = __float_as_uint(-INFINITY);
        }
        // row max with four independent 3-input max chains
        float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int c = 0; c < 32; c += 2)
            mxv[i] = fmax3(mxv[i], __uint_as_float(s[i][c]), __uint_as_float(s[i][c + 1]));
        const float mx = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3]));
        const float m_tile = mx * a.scale_log2;  // scale > 0, so max commutes with the scaling
        const bool need = (m2 == -INFINITY) || (m_tile > m2 + kRescaleThreshold);
        const float m_use = need ? fmaxf(m2, m_tile) : m2;
        const float alpha = (m2 == -INFINITY) ? 0.f : ex2(m2 - m_use);
        const float m_ref = (m_use == -INFINITY) ? 0.f : m_use;
        // probabilities p = exp2(s * scale_log2 - m_ref), two lanes of work per packed op
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(-m_ref, -m_ref);
        float2 ex0 = make_float2(0.f, 0.f), ex1 = make_float2(0.f, 0.f);  // unrounded sums
        float2 rd0 = make_float2(0.f, 0.f), rd1 = make_float2(0.f, 0.f);  // sums of the bf16 values
        // probabilities of score half hf (64 columns) packed into pk
        auto exp_half = [&](int hf, uint32_t(&pk)[32]) {
#pragma unroll
          for (int ii = 0; ii < 2; ++ii) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              const uint32_t* sr = s[hf * 2 + ii];
              const float2 x0 = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nm2);
              const float2 x1 = ffma2(make_float2(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])), sc2, nm2);
              const float2 p0 = make_float2(ex2(x0.x), ex2(x0.y));
              // one pair in kExpFmaEvery * 2 goes to the FMA pipes: the MUFU unit
              // alone (16 per cycle per SM) would bound the tile
              constexpr int kEvery = exp_fma_every<D>();
              const float2 p1 =
                  (((c >> 2) % kEvery) == kEvery - 1) ? exp2_fma2(x1) : make_float2(ex2(x1.x), ex2(x1.y));
              const uint32_t k0 = pack_bf16x2(p0.x, p0.y), k1 = pack_bf16x2(p1.x, p1.y);
              uint32_t s0 = k0, s1 = k1;  // P as the P V product takes it
              if constexpr (kDrop) {
                // keys c .. c + 3 of this 32-key word of the tile
                const uint32_t kw = keepw[hf * 2 + ii] >> c;
                const float z0 = (kw & 1u) ? a.drop_scale : 0.f;
                const float z1 = (kw & 2u) ? a.drop_scale : 0.f;
                const float z2 = (kw & 4u) ? a.drop_scale : 0.f;
                const float z3 = (kw & 8u) ? a.drop_scale : 0.f;
                s0 = pack_bf16x2(p0.x * z0, p0.y * z1);
                s1 = pack_bf16x2(p1.x * z2, p1.y * z3);
              }
              pk[ii * 16 + (c >> 1)] = s0;
              pk[ii * 16 + (c >> 1) + 1] = s1;
              ex0 = fadd2(ex0, p0);
              ex1 = fadd2(ex1, p1);
              if constexpr (D == 128) {
                // bf16 halves added to fp32 sums directly (sm_100's mixed-precision
                // add; the same sums bit for bit): 1.7% faster at d = 128, 2.7%
                // slower at d = 64, which keeps the unpack-and-add pair
                acc_bf16x2(rd0, k0);
                acc_bf16x2(rd1, k1);
              } else {
                rd0 = fadd2(rd0, make_float2(__uint_as_float(k0 << 16), __uint_as_float(k0 & 0xFFFF0000u)));
                rd1 = fadd2(rd1, make_float2(__uint_as_float(k1 << 16), __uint_as_float(k1 & 0xFFFF0000u)));
              }
            }
          }
        };
        // rescale the O accumulator when some row of this warp moved its reference.
        // The previous P.V of this tile has completed: with P over S, the scores just
        // read were issued after it and tcgen05 operations complete in order; with
        // separate P the wait for the P columns below covers it.
        const bool rescale = (kSparse ? kept_n > 0 : j > 0) && __any_sync(0xffffffffu, need);
        auto rescale_o = [&]() {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO + cc * 32, o);
          }
        };
        // separate P: both halves wait in registers for the P columns
        uint32_t pkk[kSepP ? 2 : 1][32];
        if constexpr (kSepP) {
          exp_half(0, pkk[0]);
          exp_half(1, pkk[1]);
        } else {
          // P over S in two halves: the first 64 keys' P V runs while the second
          // half's exponentials do (O is rescaled before it)
          if (rescale) rescale_o();
          exp_half(0, pkk[0]);
          tmem_st32(tS, pkk[0]);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive_warp(bar_p_half + t);
          exp_half(1, pkk[0]);
          tmem_st32(tS + 32, pkk[0]);
        }
        if constexpr (kSepP) {
          // the previous P V of this tile has read the P columns (and updated O)
          if (s_cnt > 0 && !warp_wait(bar_p_free + t, (s_cnt - 1) & 1, a.timeout_ns)) {
            if (lane == 0) record_timeout(a.status, abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          tmem_st32(tP, pkk[0]);
          tmem_st32(tP + 32, pkk[1]);
        }
        l = l * alpha + ((rd0.x + rd0.y) + (rd1.x + rd1.y));
        le = le * alpha + ((ex0.x + ex0.y) + (ex1.x + ex1.y));
        m2 = m_use;
        if constexpr (kSepP) {
          if (rescale) rescale_o();
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive_warp(bar_p_full + t);
        ++s_cnt;
        if constexpr (kSparse) ++kept_n;
      }
      if (!ok) break;

      // ---------------------------------------------------------------- epilogue
      if (!warp_wait(bar_o_done + t, tile_iter & 1, a.timeout_ns) || *abort_flag) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const SeqView se = seq_view(a, b);  // read again rather than kept live through the loop
      // a variable-length tile that runs past its sequence writes its rows itself
      const bool direct = a.cu_q != nullptr && row0 + 128 > se.lq;
      uint4* orow = reinterpret_cast<uint4*>(a.o + ((size_t)(se.qoff + row) * a.H + h) * D);
      if constexpr (L::kEarlyQ) {
        // the staging buffer is free once this group's previous TMA store has read it
        if (tid_in_group == 0) {
          bulk_wait_group_read0();
          mbar_arrive(bar_stage_free + t);
        }
        if (!warp_wait(bar_stage_free + t, tile_iter & 1, a.timeout_ns) || *abort_flag) {
          if (lane == 0) record_timeout(a.status, abort_flag);
          break;
        }
      }
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        if (kSparse ? kept_n > 0 : nkv > 0) {
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        const int box = cc >> 1;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = (cc & 1) * 4 + q4;  // 16-byte chunk within the 128-byte row
          const uint32_t addr = o_stage_u32 + box * L::kBoxBytes + r * 128 + ((chunk ^ (r & 7)) << 4);
          const float* f = reinterpret_cast<const float*>(o) + q4 * 8;
          const uint4 packed = make_uint4(pack_bf16x2(f[0] * inv_l, f[1] * inv_l), pack_bf16x2(f[2] * inv_l, f[3] * inv_l),
                                          pack_bf16x2(f[4] * inv_l, f[5] * inv_l), pack_bf16x2(f[6] * inv_l, f[7] * inv_l));
          if (!direct)
            st_shared_v4(addr, packed.x, packed.y, packed.z, packed.w);
          else if (row < se.lq)
            orow[cc * 4 + q4] = packed;
        }
      }
      if (row < se.lq) {
        const float lse = (le > 0.f) ? (m2 + __log2f(le)) * 0.69314718055994530942f : -INFINITY;
        if (a.cu_q != nullptr)
          a.lse[(size_t)h * a.total_q + se.qoff + row] = lse;
        else
          a.lse[((size_t)b * a.H + h) * a.Nq + row] = lse;
      }
      fence_proxy_async_smem();
      mbar_arrive_warp(bar_epi + t);
      bool epi_ok = true;
      if (tid_in_group == 0) {
        if (!mbar_wait(bar_epi + t, tile_iter & 1, a.timeout_ns)) {
          record_timeout(a.status, abort_flag);
          epi_ok = false;
        } else {
          if (!direct) {
            for (int bx = 0; bx < L::kBoxes; ++bx)
              tma_store_4d(&tmO, o_stage + bx * L::kBoxBytes, bx * 64, h, se.qoff + row0, se.bc);
            bulk_commit_group();
            if constexpr (!L::kEarlyQ) bulk_wait_group_read0();  // the Q tile is reloaded next
          }
          if constexpr (!L::kEarlyQ) mbar_arrive(bar_q_empty);
        }
      }
      // keep the warp converged before its next tcgen05 instruction
      if (__shfl_sync(0xffffffffu, epi_ok ? 1 : 0, 0) == 0) break;
      ++tile_iter;
    }
    if (tid_in_group == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0) {
    // this CTA takes no more items; the last CTA to finish leaves the counters at
    // zero for the next call
    __threadfence();
    if (atomicAdd(a.done_ctr, 1u) == gridDim.x - 1) {
      atomicExch(a.item_ctr, 0u);
      atomicExch(a.done_ctr, 0u);
    }
  }
}

}  // namespace

template <int D>
static fa_status launch_fwd_impl(const FwdLaunch& L0, cudaStream_t stream) {
  using L = FwdLayout<D>;
  static PerDeviceOnce attr_once;
  if (!attr_once.run([] {
        const int bytes = L::kSmemBytes;
        return cudaFuncSetAttribute(fwd_kernel<D, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    bytes) == cudaSuccess &&
               cudaFuncSetAttribute(fwd_kernel<D, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    bytes) == cudaSuccess &&
               cudaFuncSetAttribute(fwd_kernel<D, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    bytes) == cudaSuccess;
      }))
    return FA_ERR_CUDA;
  // a variable-length batch is one long batch of total rows for the TMA maps
  const bool varlen = L0.cu_q != nullptr;
  const int mB = varlen ? 1 : L0.B;
  const int mNq = varlen ? L0.total_q : L0.Nq, mNk = varlen ? L0.total_k : L0.Nk;
  CUtensorMap tq, tk, tv, to;
  if (!encode_bshd_map(&tq, L0.q, mB, mNq, L0.H, D) || !encode_bshd_map(&tk, L0.k, mB, mNk, L0.H, D) ||
      !encode_bshd_map(&tv, L0.v, mB, mNk, L0.H, D) || !encode_bshd_map(&to, L0.o, mB, mNq, L0.H, D))
    return FA_ERR_CUDA;
  FwdArgs a;
  a.lse = L0.lse;
  a.status = L0.status;
  // the item counters sit in the status block's padding (bytes 128 .. 135)
  a.item_ctr = reinterpret_cast<unsigned int*>(reinterpret_cast<uint8_t*>(L0.status) + 128);
  a.done_ctr = a.item_ctr + 1;
  a.o = static_cast<__nv_bfloat16*>(L0.o);
  a.cu_q = L0.cu_q;
  a.cu_k = L0.cu_k;
  a.total_q = L0.total_q;
  a.total_k = L0.total_k;
  a.B = L0.B;
  a.H = L0.H;
  a.Nq = L0.Nq;
  a.Nk = L0.Nk;
  a.causal = L0.causal;
  a.scale_log2 = L0.scale * 1.4426950408889634f;
  a.n_pairs = (L0.Nq + 255) / 256;
  a.n_items = a.n_pairs * L0.B * L0.H;
  a.timeout_ns = L0.timeout_ns;
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
  if (a.block_mask != nullptr && a.drop_t != 0u) return FA_ERR_UNSUPPORTED;  // no entry point combines them
  const int grid = std::min(a.n_items, num_sms() * 1);
  prof_before(stream, kKFwd);
  if (a.block_mask != nullptr)
    fwd_kernel<D, false, true><<<grid, kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, to, a);
  else if (a.drop_t != 0u)
    fwd_kernel<D, true, false><<<grid, kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, to, a);
  else
    fwd_kernel<D, false, false><<<grid, kThreads, L::kSmemBytes, stream>>>(tq, tk, tv, to, a);
  const cudaError_t err = cudaGetLastError();
  prof_after(stream, kKFwd);
  return err == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status launch_fwd(const FwdLaunch& L0, cudaStream_t stream) {
  if (L0.d == 64) return launch_fwd_impl<64>(L0, stream);
  if (L0.d == 128) return launch_fwd_impl<128>(L0, stream);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
