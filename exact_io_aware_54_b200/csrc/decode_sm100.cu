// decode_sm100.cu -- split-KV decode over a ragged, packed KV cache (B200, sm_100a).
//
// What it computes: for each sequence b and head h, the single new query row
// attends to that sequence's L_b cached keys,
//     o = sum_j softmax_j(scale * q . k_j) v_j,   lse = ln sum_j exp(scale * q . k_j).
// The keys are cut into chunks; each CTA reduces its chunk to the running
// (m, l, u) state ("FlashAttention saves IO, not N^2 work", section 2) and the
// chunk states are merged with the block-merge rule of sections 3 and 7 of the
// same page.  Decode reads the whole KV history once, so this path is bound by
// HBM bandwidth (section 6 of that page: single-request and batched decode).
//
// B200 design
//  * Grid (split, head group, sequence).  A head group is up to 8 heads; the
//    CTA has one warp per head plus one producer warp.  The CTAs of one
//    (sequence, head group) share its keys dynamically: each producer takes the
//    next chunk of keys from a per-(sequence, group) atomic counter whenever it
//    has issued the previous one, and its consumers fold every chunk the CTA
//    takes into one running state (the (m, l, u) state of any set of keys is
//    order-independent), so each CTA still leaves exactly one partial state.  A
//    static split of one wave left the CTAs that the memory system served last
//    streaming alone at the end (per-SM busy time ranged over 3.5x at one
//    request of 8192 keys, H = 32); with shared chunks every SM stays busy until
//    the keys run out.
//  * For every key of its chunk the head group's K and V slices are contiguous
//    (8 heads x d bf16), so the producer moves them with plain bulk copies
//    (cp.async.bulk) into a ring of shared-memory stages of 8 keys, completion
//    counted on mbarriers.  Rows are padded by 64 bytes so the consumer reads are
//    free of bank conflicts.
//  * Consumer warp = head.  Lane = (key slot t in 0..7) x (part p in 0..3); part
//    p owns 16-byte chunks p, p+4, ... of the head dimension.  Scores need two
//    shuffle levels, the stage max three; every lane keeps a partial u over the
//    keys of its slot, summed across slots once at the end.
//  * The producer writes each stage's first key and key count into a header
//    beside the stage; a header with no keys tells the consumers that the
//    counter ran out.  The last producer of a (sequence, group) to run out --
//    found with a second ticket -- resets the counter, so counters are zero
//    between calls.
//  * The last warp of each (sequence, head) to finish its CTA's state -- found with
//    an atomic ticket -- merges the CTAs' states and writes o and lse, then resets
//    the ticket, so tickets are zero between calls.  A sequence served by a single
//    CTA skips the partial-state round trip.
//  * Given the number of rows of a packed cache, every sequence's offsets are
//    checked against it first; a sequence outside the buffers is skipped and
//    recorded in the status word.
//  * Paged caches (K and V in pages of page_size keys, a block table per
//    sequence) only change where the producer reads a key's row from; every page
//    index is checked against the number of pages (a bad one is recorded in the
//    status word and read as page 0, so no copy leaves the cache).
#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr int kHeadsPerCta = 8;
constexpr int kKeysPerStage = 8;
constexpr int kThreads = (kHeadsPerCta + 1) * 32;
// Two CTAs per SM, each with a ring of about 100 KB of copies in flight.  (One CTA
// per SM with a ring twice as deep halves the chunk states the merge reads, but
// eight consumer warps per SM then fall behind: measured 17% slower at one request
// of 8192 keys and 25% slower on the 64-request batch.)
#ifndef FA_DEC_CTAS_PER_SM
#define FA_DEC_CTAS_PER_SM 2
#endif
constexpr int kCtasPerSm = FA_DEC_CTAS_PER_SM;
// states the merge loads per round trip (registers allow more with one CTA per SM)
constexpr int kMergeBatch = kCtasPerSm == 1 ? 32 : 16;

template <int D>
struct DecLayout {
  static constexpr int kRowBytes = kHeadsPerCta * D * 2;  // one key, all heads of the group
  static constexpr int kRowStride = kRowBytes + 64;       // padded
  static constexpr int kStageBytes = 2 * kKeysPerStage * kRowStride;  // K rows then V rows
  static constexpr int kStages = (D == 128 ? 6 : 12) / kCtasPerSm;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kOffHdr = kOffBar + 2 * kStages * 8 + 64;  // int2 (first key, keys) per stage
  static constexpr int kSmemBytes = kOffHdr + kStages * 8 + 128;
  static constexpr int kChunks = D / 32;  // 16-byte chunks per lane
};

struct DecArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* cu;
  const int32_t* block_table;  // paged cache when not null
  const int32_t* seqlens;
  int page_size, max_pages, num_pages;
  int total_kv;  // packed cache rows, checked against the offsets when >= 0
  __nv_bfloat16* o;
  float* lse;
  int* status;
  unsigned int* tickets;      // [B * H] merge tickets
  unsigned int* grab;         // [B * groups] next chunk of keys to hand out
  unsigned int* grab_done;    // [B * groups] producers that found no chunk left
  float* part_ml;
  float* part_u;
  int B, H, max_seqlen_k;
  int gchunk, splits, groups;  // keys per chunk handed out, CTAs per (sequence, group), groups
  float scale_log2;
  int check_args;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void bf16x8_to_f32(uint32_t a, uint32_t b, uint32_t c, uint32_t d, float (&f)[8]) {
  f[0] = __uint_as_float(a << 16);
  f[1] = __uint_as_float(a & 0xFFFF0000u);
  f[2] = __uint_as_float(b << 16);
  f[3] = __uint_as_float(b & 0xFFFF0000u);
  f[4] = __uint_as_float(c << 16);
  f[5] = __uint_as_float(c & 0xFFFF0000u);
  f[6] = __uint_as_float(d << 16);
  f[7] = __uint_as_float(d & 0xFFFF0000u);
}

template <int D>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_kernel(const DecArgs a) {
  using L = DecLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* empty = full + L::kStages;
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L::kOffBar + 2 * L::kStages * 8);
  // flags[0]: abort

  const int split = blockIdx.x, group = blockIdx.y, b = blockIdx.z;
  const int h0 = group * kHeadsPerCta;
  const int nh = min(kHeadsPerCta, a.H - h0);
  if (a.check_args && *reinterpret_cast<volatile int*>(a.status) == kStatusBadArg) return;

  const bool paged = a.block_table != nullptr;
  const int start = paged ? 0 : a.cu[b];
  if (!paged && a.total_kv >= 0) {
    // rows start .. end - 1 must lie inside k and v; otherwise every CTA of this
    // sequence leaves it alone (nothing is read or written for it)
    const int end = a.cu[b + 1];
    if (start < 0 || end < start || end > a.total_kv) {
      if (split == 0 && group == 0 && threadIdx.x == 0) atomicExch(a.status, kStatusBadArg);
      return;
    }
  }
  int len = paged ? a.seqlens[b] : a.cu[b + 1] - start;
  len = max(0, min(len, a.max_seqlen_k));
  // CTAs of this (sequence, group) that take part: at most one per chunk
  const int nsplit = min(a.splits, (len + a.gchunk - 1) / a.gchunk);
  const uint32_t warp = warp_id(), lane = lane_id();

  if (len == 0) {
    // empty history: o = 0, lse = -inf (written once, by chunk 0)
    if (split == 0 && (int)warp < nh) {
      const int h = h0 + warp;
      for (int c = lane; c < D; c += 32) a.o[((size_t)b * a.H + h) * D + c] = __float2bfloat16(0.f);
      if (lane == 0) a.lse[(size_t)b * a.H + h] = -INFINITY;
    }
    return;
  }
  if (split >= nsplit) return;
  int2* hdr = reinterpret_cast<int2*>(smem + L::kOffHdr);
  const size_t bg = (size_t)b * a.groups + group;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kHeadsPerCta);
    }
    flags[0] = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  __syncthreads();

  const size_t row_elems = (size_t)a.H * D;          // elements per key row of k / v
  const uint32_t copy_bytes = (uint32_t)nh * D * 2;  // this group's slice of one key row

  if (warp == kHeadsPerCta) {
    // ------------------------------------------------------------------ producer warp
    // The first chunk of CTA `split` is chunk `split` (there is one per CTA that
    // takes part), so no counter round trip delays the first copies; later chunks
    // come from the counter (nsplit + the value taken).  Lane 0 takes the next one
    // while the current chunk's copies are issued; every chunk taken is issued.
    unsigned int next = (unsigned)split;
    int issued = 0;  // stages issued (ring position)
    bool ok = true;
    while (ok) {
      const int c = (int)__shfl_sync(0xffffffffu, next, 0);
      const bool more = (long long)c * a.gchunk < len;
      if (more && lane == 0) next = (unsigned)nsplit + atomicAdd(a.grab + bg, 1u);
      for (int st = 0; ok; ++st) {
        const int key0 = more ? c * a.gchunk + st * kKeysPerStage : 0;
        if (more && (st * kKeysPerStage >= a.gchunk || key0 >= len)) break;
        const int nk = more ? min(kKeysPerStage, len - key0) : -1;  // -1: no chunk left
        const int slot = issued % L::kStages;
        const uint32_t phase = (issued / L::kStages) & 1;
        if (lane == 0) {
          ok = mbar_wait(empty + slot, phase ^ 1, a.timeout_ns) && !flags[0];
          if (ok) {
            hdr[slot] = make_int2(key0, nk);
            if (more)
              mbar_arrive_expect_tx(full + slot, 2u * nk * copy_bytes);
            else
              mbar_arrive(full + slot);  // the header alone: no copies
          } else {
            flags[0] = 1;
            atomicCAS(a.status, 0, kStatusTimeout);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++issued;
        if (!more) break;
        if (lane < 2 * kKeysPerStage) {
          const int t = lane & (kKeysPerStage - 1);
          const int is_v = lane >= kKeysPerStage;
          const int key = key0 + t;
          if (t < nk) {
            size_t row = (size_t)start + key;
            if (paged) {
              int page = a.block_table[(size_t)b * a.max_pages + key / a.page_size];
              if (page < 0 || page >= a.num_pages) {  // never read outside the cache
                atomicExch(a.status, kStatusBadArg);
                page = 0;
              }
              row = (size_t)page * a.page_size + key % a.page_size;
            }
            const __nv_bfloat16* src = (is_v ? a.v : a.k) + row * row_elems + (size_t)h0 * D;
            uint8_t* dst = smem + slot * L::kStageBytes + is_v * kKeysPerStage * L::kRowStride + t * L::kRowStride;
            bulk_load(dst, src, copy_bytes, full + slot);
          }
        }
      }
      if (!more) break;
    }
    if (lane == 0) {
      if (ok) {
        // this producer takes no more chunks; the last of the (sequence, group) to
        // get here resets the counter for the next call (every other producer has
        // made its final take by then: each takes before it counts itself here)
        __threadfence();
        if (atomicAdd(a.grab_done + bg, 1u) == (unsigned)(nsplit - 1)) {
          atomicExch(a.grab + bg, 0u);
          atomicExch(a.grab_done + bg, 0u);
        }
      } else {
        // on an early exit, let the copies already issued land before the CTA retires
        for (int s2 = max(0, issued - L::kStages); s2 < issued; ++s2)
          (void)mbar_wait(full + (s2 % L::kStages), (s2 / L::kStages) & 1, a.timeout_ns);
      }
    }
    return;
  }

  // -------------------------------------------------------------------- consumer warps
  const int hw = warp;  // head within the group
  const bool head_ok = hw < nh;
  const int h = h0 + hw;
  const int t = lane >> 2, p = lane & 3;

  // q chunks owned by this lane, pre-scaled into the log2 domain
  float qf[L::kChunks][8];
#pragma unroll
  for (int i = 0; i < L::kChunks; ++i) {
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (head_ok) raw = *reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.H + h) * D + (p + 4 * i) * 8);
    bf16x8_to_f32(raw.x, raw.y, raw.z, raw.w, qf[i]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[i][e] *= a.scale_log2;
  }
  float u[L::kChunks][8];
#pragma unroll
  for (int i = 0; i < L::kChunks; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) u[i][e] = 0.f;
  float m = -INFINITY, l = 0.f;
  bool ok = true;

  for (int s = 0;; ++s) {
    const int slot = s % L::kStages;
    bool got = true;
    if (lane == 0) got = mbar_wait(full + slot, (s / L::kStages) & 1, a.timeout_ns) && !flags[0];
    got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
    if (!got) {
      if (lane == 0) {
        flags[0] = 1;
        atomicCAS(a.status, 0, kStatusTimeout);
      }
      ok = false;
      break;
    }
    const int nk = hdr[slot].y;
    if (nk < 0) break;  // no chunk left for this CTA
    const bool valid = head_ok && t < nk;
    const uint32_t kaddr = smem_u32(smem + slot * L::kStageBytes + t * L::kRowStride + hw * D * 2);
    const uint32_t vaddr = kaddr + kKeysPerStage * L::kRowStride;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < L::kChunks; ++i) {
      uint32_t r0, r1, r2, r3;
      ld_shared_v4(kaddr + (p + 4 * i) * 16, r0, r1, r2, r3);
      float kf[8];
      bf16x8_to_f32(r0, r1, r2, r3, kf);
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(qf[i][e], kf[e], dot);
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    const float x = valid ? dot : -INFINITY;
    float mx = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float m_new = fmaxf(m, mx);
    const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = (m == -INFINITY) ? 0.f : ex2(m - m_ref);
    const float pw = ex2(x - m_ref);
    l = l * alpha + pw;
#pragma unroll
    for (int i = 0; i < L::kChunks; ++i) {
      uint32_t r0, r1, r2, r3;
      ld_shared_v4(vaddr + (p + 4 * i) * 16, r0, r1, r2, r3);
      float vf[8];
      bf16x8_to_f32(r0, r1, r2, r3, vf);
#pragma unroll
      for (int e = 0; e < 8; ++e) u[i][e] = valid ? fmaf(pw, vf[e], u[i][e] * alpha) : u[i][e] * alpha;
    }
    m = m_new;
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + slot);
  }

  // combine the 8 key slots: every lane ends with the sums for its own chunks
  l += __shfl_xor_sync(0xffffffffu, l, 4);
  l += __shfl_xor_sync(0xffffffffu, l, 8);
  l += __shfl_xor_sync(0xffffffffu, l, 16);
#pragma unroll
  for (int i = 0; i < L::kChunks; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float x = u[i][e];
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      x += __shfl_xor_sync(0xffffffffu, x, 16);
      u[i][e] = x;
    }
  if (!ok) return;

  const size_t bh = (size_t)b * a.H + h;
  if (nsplit == 1) {
    // the whole history was one chunk: finish here
    if (head_ok && t == 0) {
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
      for (int i = 0; i < L::kChunks; ++i) {
        uint4 w;
        w.x = pack_bf16x2(u[i][0] * inv, u[i][1] * inv);
        w.y = pack_bf16x2(u[i][2] * inv, u[i][3] * inv);
        w.z = pack_bf16x2(u[i][4] * inv, u[i][5] * inv);
        w.w = pack_bf16x2(u[i][6] * inv, u[i][7] * inv);
        *reinterpret_cast<uint4*>(a.o + bh * D + (p + 4 * i) * 8) = w;
      }
      if (p == 0) a.lse[bh] = (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
    return;
  }

  // write this chunk's state; the last chunk of (b, h) to finish merges them all
  if (!head_ok) return;
  if (t == 0) {
    float* pu = a.part_u + (bh * a.splits + split) * D;
#pragma unroll
    for (int i = 0; i < L::kChunks; ++i) {
      float4* dst = reinterpret_cast<float4*>(pu + (p + 4 * i) * 8);
      __stcg(dst, make_float4(u[i][0], u[i][1], u[i][2], u[i][3]));
      __stcg(dst + 1, make_float4(u[i][4], u[i][5], u[i][6], u[i][7]));
    }
    if (p == 0) __stcg(reinterpret_cast<float2*>(a.part_ml) + bh * a.splits + split, make_float2(m, l));
  }
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) last = (atomicAdd(a.tickets + bh, 1u) == (unsigned)(nsplit - 1)) ? 1 : 0;
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();

  // ------------------------------------------------------------------ merge (last state of b, h)
  // The states are read kMergeBatch at a time, every load of a batch issued before
  // any is used, with a running reference max: one L2 round trip per batch.  Lane
  // i weighs state s0 + i; each lane sums the u of every state over its own kPerLane
  // columns, with the weights passed round by shuffles.
  constexpr int kPerLane = D / 32;
  const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + bh * a.splits;
  const float* pu = a.part_u + bh * a.splits * D + lane * kPerLane;
  float M = -INFINITY, Lsum = 0.f, U[kPerLane];
#pragma unroll
  for (int e = 0; e < kPerLane; ++e) U[e] = 0.f;
  for (int s0 = 0; s0 < nsplit; s0 += kMergeBatch) {
    const int s_own = s0 + (int)(lane % kMergeBatch);
    const float2 st = (lane < (uint32_t)kMergeBatch && s_own < nsplit) ? __ldcg(ml + s_own)
                                                                       : make_float2(-INFINITY, 0.f);
    float uu[kMergeBatch][kPerLane];
#pragma unroll
    for (int i = 0; i < kMergeBatch; ++i) {
      const int s = min(s0 + i, nsplit - 1);
      if constexpr (kPerLane == 4) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(pu + (size_t)s * D));
        uu[i][0] = x.x;
        uu[i][1] = x.y;
        uu[i][2] = x.z;
        uu[i][3] = x.w;
      } else {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(pu + (size_t)s * D));
        uu[i][0] = x.x;
        uu[i][1] = x.y;
      }
    }
    float mb = st.x;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
    const float M_new = fmaxf(M, mb);
    const float M_ref = (M_new == -INFINITY) ? 0.f : M_new;
    const float keep = (M == -INFINITY) ? 0.f : ex2(M - M_ref);  // rescale what was summed so far
    Lsum *= keep;
#pragma unroll
    for (int e = 0; e < kPerLane; ++e) U[e] *= keep;
    const float w = (st.x == -INFINITY) ? 0.f : ex2(st.x - M_ref);  // 0 past the last state
    Lsum = fmaf(w, st.y, Lsum);
#pragma unroll
    for (int i = 0; i < kMergeBatch; ++i) {
      const float wi = __shfl_sync(0xffffffffu, w, i);
#pragma unroll
      for (int e = 0; e < kPerLane; ++e) U[e] = fmaf(wi, uu[i][e], U[e]);
    }
    M = M_new;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, off);
  const float inv = (Lsum > 0.f) ? 1.f / Lsum : 0.f;
  __nv_bfloat16* out = a.o + bh * D + lane * kPerLane;
#pragma unroll
  for (int e = 0; e < kPerLane; e += 2)
    *reinterpret_cast<uint32_t*>(out + e) = pack_bf16x2(U[e] * inv, U[e + 1] * inv);
  if (lane == 0) {
    a.lse[bh] = (Lsum > 0.f) ? (M + __log2f(Lsum)) * 0.69314718055994530942f : -INFINITY;
    a.tickets[bh] = 0u;  // every chunk of (b, h) has arrived: ready for the next call
  }
}

// Optional argument check of cu_seqlens (FA_CHECKS=1).
__global__ void check_cu_seqlens_kernel(const int32_t* cu, int B, int max_seqlen_k, int* status) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b <= B; b += gridDim.x * blockDim.x) {
    bool bad = false;
    if (b == 0) bad = cu[0] != 0;
    else {
      const int L = cu[b] - cu[b - 1];
      bad = L < 0 || L > max_seqlen_k;
    }
    if (bad) atomicExch(status, kStatusBadArg);
  }
}

}  // namespace

DecodePlan decode_plan(int B, int H, int max_seqlen_k, int d, int num_splits) {
  (void)d;
  DecodePlan p;
  p.heads_per_group = std::min(H, kHeadsPerCta);
  p.groups = (H + kHeadsPerCta - 1) / kHeadsPerCta;
  const int maxL = std::max(max_seqlen_k, 1);
  auto roundup8 = [](long long x) { return (int)(((x + 7) / 8) * 8); };
  int chunk;
  if (num_splits > 0) {
    const int s = std::max(1, std::min(num_splits, (maxL + 7) / 8));
    chunk = roundup8((maxL + s - 1) / s);
  } else {
    const long long slots = (long long)num_sms() * kCtasPerSm;
    const long long work = (long long)B * maxL * p.groups;
    chunk = roundup8((work + slots * 16 - 1) / (slots * 16));  // ~16 waves if all sequences are full
    if (chunk < 256) {
      // a small problem: spread it over one wave of CTAs
      const long long units = (long long)B * p.groups;
      const long long s = std::max(1LL, (slots + units - 1) / units);
      chunk = roundup8((maxL + s - 1) / s);
    }
  }
  chunk = std::max(chunk, 8);
  int splits = (maxL + chunk - 1) / chunk;
  while (splits > 4096) {  // bound the partial-state workspace
    chunk *= 2;
    splits = (maxL + chunk - 1) / chunk;
  }
  p.chunk = chunk;
  p.splits = splits;
  // chunks handed out: about an eighth of a CTA's even share of the keys, so the
  // CTAs of a (sequence, group) can even out how fast each is served, but at
  // least two stages (one counter round trip hides behind two stages of copies)
  p.gchunk = std::min(256, std::max(16, roundup8(chunk / 8)));
  return p;
}

namespace {
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
}  // namespace

size_t decode_workspace_bytes(int B, int H, int d, const DecodePlan& plan) {
  size_t bytes = kStatusBytes + kDecodeSyncBytes;
  if ((size_t)B * H > kDecodeFixedTickets) bytes += up256(sizeof(unsigned) * 3 * (size_t)B * H);
  bytes += up256(sizeof(float) * 2 * (size_t)B * H * plan.splits);
  bytes += up256(sizeof(float) * (size_t)d * B * H * plan.splits);
  return bytes;
}

void decode_carve(uint8_t* ws, int B, int H, int d, const DecodePlan& plan, DecodeLaunch& a) {
  a.status = reinterpret_cast<int*>(ws);
  unsigned* sync = reinterpret_cast<unsigned*>(ws + kStatusBytes);
  size_t off = kStatusBytes + kDecodeSyncBytes;
  a.part_ml = reinterpret_cast<float*>(ws + off);
  off += up256(sizeof(float) * 2 * (size_t)B * H * plan.splits);
  a.part_u = reinterpret_cast<float*>(ws + off);
  off += up256(sizeof(float) * (size_t)d * B * H * plan.splits);
  size_t n = kDecodeFixedTickets;
  a.clear_ptr = nullptr;
  a.clear_bytes = 0;
  if ((size_t)B * H > kDecodeFixedTickets) {
    // too many (sequence, head) pairs for the fixed region: a region of this call's
    // own, cleared before the launch
    sync = reinterpret_cast<unsigned*>(ws + off);
    n = (size_t)B * H;
    a.clear_ptr = sync;
    a.clear_bytes = sizeof(unsigned) * 3 * n;
  }
  a.tickets = sync;
  a.grab = sync + n;
  a.grab_done = sync + 2 * n;
}

template <int D>
static fa_status launch_decode_impl(const DecodeLaunch& L0, cudaStream_t stream) {
  using L = DecLayout<D>;
  static PerDeviceOnce attr_once;
  if (!attr_once.run([] {
        return cudaFuncSetAttribute(decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kSmemBytes) == cudaSuccess;
      }))
    return FA_ERR_CUDA;
  DecArgs a;
  a.q = static_cast<const __nv_bfloat16*>(L0.q);
  a.k = static_cast<const __nv_bfloat16*>(L0.k);
  a.v = static_cast<const __nv_bfloat16*>(L0.v);
  a.cu = L0.cu_seqlens;
  a.block_table = L0.block_table;
  a.seqlens = L0.seqlens;
  a.page_size = L0.page_size;
  a.max_pages = L0.max_pages;
  a.num_pages = L0.num_pages;
  a.total_kv = L0.total_kv;
  a.o = static_cast<__nv_bfloat16*>(L0.o);
  a.lse = L0.lse;
  a.status = L0.status;
  a.tickets = L0.tickets;
  a.grab = L0.grab;
  a.grab_done = L0.grab_done;
  a.part_ml = L0.part_ml;
  a.part_u = L0.part_u;
  a.B = L0.B;
  a.H = L0.H;
  a.max_seqlen_k = L0.max_seqlen_k;
  a.gchunk = L0.plan.gchunk;
  a.splits = L0.plan.splits;
  a.groups = L0.plan.groups;
  a.scale_log2 = L0.scale * 1.4426950408889634f;
  a.check_args = L0.check_args;
  a.timeout_ns = L0.timeout_ns;
  if (L0.clear_bytes) {
    if (cudaMemsetAsync(L0.clear_ptr, 0, L0.clear_bytes, stream) != cudaSuccess) return FA_ERR_CUDA;
  }
  if (L0.check_args && !L0.block_table) {
    prof_before(stream, kKDecodeCheck);
    check_cu_seqlens_kernel<<<(L0.B + 256) / 256, 256, 0, stream>>>(L0.cu_seqlens, L0.B, L0.max_seqlen_k,
                                                                      L0.status);
    const cudaError_t err = cudaGetLastError();
    prof_after(stream, kKDecodeCheck);
    if (err != cudaSuccess) return FA_ERR_CUDA;
  }
  dim3 grid(L0.plan.splits, L0.plan.groups, L0.B);
  prof_before(stream, kKDecode);
  decode_kernel<D><<<grid, kThreads, L::kSmemBytes, stream>>>(a);
  const cudaError_t err = cudaGetLastError();
  prof_after(stream, kKDecode);
  return err == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status launch_decode(const DecodeLaunch& L0, cudaStream_t stream) {
  if (L0.d == 64) return launch_decode_impl<64>(L0, stream);
  if (L0.d == 128) return launch_decode_impl<128>(L0, stream);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
