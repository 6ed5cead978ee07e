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
//  * Grid (head group, split, sequence).  A head group is the heads whose slices
//    of one key row make 256 contiguous bytes: one head of d = 128, two of
//    d = 64.  Eight consumer warps share the group's keys (each takes 8 keys of
//    every stage), plus one producer warp.  Few heads per CTA keep the number of
//    partial states per head small -- one per CTA that serves it, about ten at one
//    request of 8192 keys, H = 32 -- so the last arrival merges them in one L2
//    round trip.  (Eight heads per CTA left 74 states per head and a merge of five
//    dependent round trips at the end of every call.)
//  * The CTAs of one (sequence, head group) share its keys dynamically: each
//    producer takes the next chunk of keys from a per-(sequence, group) atomic
//    counter whenever it has issued the previous one, and its consumers fold every
//    chunk the CTA takes into one running state (the (m, l, u) state of any set of
//    keys is order-independent), so each CTA still leaves exactly one partial
//    state.  A static split of one wave left the CTAs that the memory system
//    served last streaming alone at the end; with shared chunks every SM stays
//    busy until the keys run out.
//  * For every key the group's K and V slices are contiguous, so the producer
//    moves them with plain bulk copies (cp.async.bulk) into a ring of
//    shared-memory stages, completion counted on mbarriers.  Rows are padded by 16
//    bytes: the eight rows that a quarter-warp reads then start four banks apart,
//    so the consumer reads are free of bank conflicts.
//  * Consumer warp = (head, 8 keys of the stage).  Lane = (part p in 0..3) x (key
//    slot t in 0..7); part p owns 16-byte chunks p, p+4, ... of the head
//    dimension.  Scores need two shuffle levels, the stage max three; every lane
//    keeps a partial u over the keys of its slot, summed across slots at the end,
//    and the warps of one head combine their states through shared memory.
//  * The producer writes each stage's first key and key count into a header
//    beside the stage; a header with no keys tells the consumers that the
//    counter ran out.  The last producer of a (sequence, group) to run out --
//    found with a second ticket -- resets the counter, so counters are zero
//    between calls.
//  * The last CTA of each (sequence, head) to finish its state -- found with an
//    atomic ticket -- merges the CTAs' states and writes o and lse, then resets
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

constexpr int kConsumers = 8;  // consumer warps per CTA
constexpr int kThreads = (kConsumers + 1) * 32;
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

// Two ways to move the keys.  Packed caches (kTiled): TMA tensor tiles, one box of
// 64 columns x kKeysPerStage keys per (head, half of a head's 128-byte column
// blocks), 128-byte swizzled in shared memory, with one head (d = 128) or two
// (d = 64) per CTA.  Paged caches, whose pages may hold any number of keys: one
// bulk copy per key of the contiguous slice of eight heads, into padded rows (a
// copy has a fixed cost of tens of cycles, so slices of 256 bytes would leave the
// copy engine, not HBM, as the bound: measured 2.5x slower).
template <int D, bool kTiled>
struct DecLayout {
  static constexpr int kHeads = kTiled ? 256 / (2 * D) : 8;    // heads per CTA
  static constexpr int kWarpsPerHead = kConsumers / kHeads;    // consumer warps sharing one head's keys
  static constexpr int kKeysPerStage = 8 * kWarpsPerHead;      // 8 keys per consumer warp and stage
  static constexpr int kRowBytes = kHeads * D * 2;             // one key, all heads of the group
  // bulk copies: rows padded by 16 bytes, so the eight rows a quarter-warp reads
  // start four banks apart; tiles: dense 128-byte rows, swizzled
  static constexpr int kRowStride = kTiled ? kRowBytes : kRowBytes + 16;
  static constexpr int kBoxBytes = kKeysPerStage * 128;        // tiles: one (head, 64-column) box
  static constexpr int kStageBytes = 2 * kKeysPerStage * kRowStride;  // K rows then V rows
  static constexpr int kStages = (D == 128 ? 6 : 12) / kCtasPerSm;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kOffHdr = kOffBar + 2 * kStages * 8 + 64;  // int4 (first key, keys, first row) per stage
  static constexpr int kOffComb = kOffHdr + kStages * 16;
  static constexpr int kCombFloats = D + 4;                       // per consumer warp: m, l, -, -, u[D]
  static constexpr int kSmemBytes = kOffComb + kConsumers * kCombFloats * 4 + 1024;  // + alignment slack
  static constexpr int kChunks = D / 32;  // 16-byte chunks per lane
  static_assert(!kTiled || (kStageBytes % 1024 == 0 && kBoxBytes % 1024 == 0),
                "swizzled boxes start on 1024-byte boundaries");
  // byte offset of 16-byte chunk c of head hw's slice of key row `row`, from the
  // start of the stage's K (or V) rows
  __device__ static __forceinline__ uint32_t chunk_off(int row, int hw, int c) {
    if constexpr (kTiled)
      return (hw * (D / 64) + (c >> 3)) * kBoxBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4);
    else
      return row * kRowStride + hw * D * 2 + c * 16;
  }
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

// tmK / tmV: the packed cache as [rows, H, D] tensors (kTiled only).
template <int D, bool kTiled>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const DecArgs a) {
  using L = DecLayout<D, kTiled>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* empty = full + L::kStages;
  volatile int* flags = reinterpret_cast<volatile int*>(smem + L::kOffBar + 2 * L::kStages * 8);
  // flags[0]: abort

  // grid (group, split, sequence): consecutive CTAs serve different head groups, so
  // the CTAs of one group spread over the whole GPU instead of sitting side by side
  // (measured: one request of 8192 keys 32.8 -> 30.9 us, the 64-request batch 1%)
  const int group = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int h0 = group * L::kHeads;
  const int nh = min(L::kHeads, a.H - h0);
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
  int4* hdr = reinterpret_cast<int4*>(smem + L::kOffHdr);
  const size_t bg = (size_t)b * a.groups + group;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kConsumers);
    }
    flags[0] = 0;
    if constexpr (kTiled) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  __syncthreads();

  const size_t row_elems = (size_t)a.H * D;          // elements per key row of k / v
  const uint32_t copy_bytes = (uint32_t)nh * D * 2;  // this group's slice of one key row

  if (warp == kConsumers) {
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
        const int key0 = more ? c * a.gchunk + st * L::kKeysPerStage : 0;
        if (more && (st * L::kKeysPerStage >= a.gchunk || key0 >= len)) break;
        const int nk = more ? min(L::kKeysPerStage, len - key0) : -1;  // -1: no chunk left
        const int slot = issued % L::kStages;
        const uint32_t phase = (issued / L::kStages) & 1;
        if (lane == 0) {
          ok = mbar_wait(empty + slot, phase ^ 1, a.timeout_ns) && !flags[0];
          if (ok) {
            // tiles: the stage's box rows end at its last key, so they never reach
            // past the sequence (rows before it belong to earlier sequences or, below
            // row 0, are filled with zeros); the keys are the last nk rows
            const int lo = kTiled && more ? L::kKeysPerStage - nk : 0;
            hdr[slot] = make_int4(key0, nk, lo, 0);
            if (!more) {
              mbar_arrive(full + slot);  // the header alone: no copies
            } else if constexpr (kTiled) {
              const int y = start + key0 + nk - L::kKeysPerStage;
              mbar_arrive_expect_tx(full + slot, 2u * nh * (D / 64) * L::kBoxBytes);
              uint8_t* dst = smem + slot * L::kStageBytes;
              for (int hh = 0; hh < nh; ++hh)
                for (int half = 0; half < D / 64; ++half) {
                  uint8_t* box = dst + (hh * (D / 64) + half) * L::kBoxBytes;
                  tma_load_3d(box, &tmK, full + slot, half * 64, h0 + hh, y);
                  tma_load_3d(box + L::kKeysPerStage * L::kRowBytes, &tmV, full + slot, half * 64, h0 + hh, y);
                }
            } else {
              mbar_arrive_expect_tx(full + slot, 2u * nk * copy_bytes);
            }
          } else {
            flags[0] = 1;
            atomicCAS(a.status, 0, kStatusTimeout);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++issued;
        if (!more) break;
        if constexpr (!kTiled) {  // (tiles: lane 0 issued the stage above)
          // copy ci < kKeysPerStage: K row of key key0 + ci, then the V rows
          for (int ci = lane; ci < 2 * L::kKeysPerStage; ci += 32) {
            const int is_v = ci >= L::kKeysPerStage;
            const int t = ci - is_v * L::kKeysPerStage;
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
              uint8_t* dst = smem + slot * L::kStageBytes + (is_v * L::kKeysPerStage + t) * L::kRowStride;
              bulk_load(dst, src, copy_bytes, full + slot);
            }
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
  const int hw = warp / L::kWarpsPerHead;  // head within the group
  const int ks = warp % L::kWarpsPerHead;  // this warp's 8 keys of every stage: ks * 8 ..
  const bool head_ok = hw < nh;
  const int h = h0 + hw;
  const int t = lane & 7, p = lane >> 3;

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
      break;
    }
    const int4 hd = hdr[slot];
    const int nk = hd.y;
    if (nk < 0) break;  // no chunk left for this CTA
    const int row = ks * 8 + t;
    const bool valid = head_ok && row >= hd.z && row < hd.z + nk;
    const uint32_t kaddr = smem_u32(smem + slot * L::kStageBytes);
    const uint32_t vaddr = kaddr + L::kKeysPerStage * L::kRowStride;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < L::kChunks; ++i) {
      uint32_t r0, r1, r2, r3;
      ld_shared_v4(kaddr + L::chunk_off(row, hw, p + 4 * i), r0, r1, r2, r3);
      float kf[8];
      bf16x8_to_f32(r0, r1, r2, r3, kf);
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(qf[i][e], kf[e], dot);
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 8);
    dot += __shfl_xor_sync(0xffffffffu, dot, 16);
    const float x = valid ? dot : -INFINITY;
    float mx = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    const float m_new = fmaxf(m, mx);
    const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = (m == -INFINITY) ? 0.f : ex2(m - m_ref);
    const float pw = ex2(x - m_ref);
    l = l * alpha + pw;
#pragma unroll
    for (int i = 0; i < L::kChunks; ++i) {
      uint32_t r0, r1, r2, r3;
      ld_shared_v4(vaddr + L::chunk_off(row, hw, p + 4 * i), r0, r1, r2, r3);
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
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  l += __shfl_xor_sync(0xffffffffu, l, 4);
#pragma unroll
  for (int i = 0; i < L::kChunks; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float x = u[i][e];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      u[i][e] = x;
    }

  // combine the warps of one head through shared memory; from here on lane i holds
  // columns i * kPerLane .. of the CTA's state (M, Lsum, U)
  constexpr int kPerLane = D / 32;
  float* comb = reinterpret_cast<float*>(smem + L::kOffComb);
  float* mine = comb + warp * L::kCombFloats;
  if (t == 0) {
#pragma unroll
    for (int i = 0; i < L::kChunks; ++i) {
      float4* dst = reinterpret_cast<float4*>(mine + 4 + (p + 4 * i) * 8);
      dst[0] = make_float4(u[i][0], u[i][1], u[i][2], u[i][3]);
      dst[1] = make_float4(u[i][4], u[i][5], u[i][6], u[i][7]);
    }
    if (p == 0) {
      mine[0] = m;
      mine[1] = l;
    }
  }
  static_assert(L::kWarpsPerHead == 1 || L::kHeads <= 2, "one named barrier per head of the group");
  if constexpr (L::kWarpsPerHead == 1)
    __syncwarp();
  else if (hw == 0)
    asm volatile("bar.sync 1, %0;" ::"n"(L::kWarpsPerHead * 32) : "memory");
  else
    asm volatile("bar.sync 2, %0;" ::"n"(L::kWarpsPerHead * 32) : "memory");
  if (flags[0] || ks != 0 || !head_ok) return;  // a wait gave up, or another warp finishes this head
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < L::kWarpsPerHead; ++w) M = fmaxf(M, comb[(warp + w) * L::kCombFloats]);
  const float M_ref0 = (M == -INFINITY) ? 0.f : M;
  float Lsum = 0.f, U[kPerLane];
#pragma unroll
  for (int e = 0; e < kPerLane; ++e) U[e] = 0.f;
#pragma unroll
  for (int w = 0; w < L::kWarpsPerHead; ++w) {
    const float* st = comb + (warp + w) * L::kCombFloats;
    const float mw = st[0];
    const float wt = (mw == -INFINITY) ? 0.f : ex2(mw - M_ref0);
    Lsum = fmaf(wt, st[1], Lsum);
#pragma unroll
    for (int e = 0; e < kPerLane; ++e) U[e] = fmaf(wt, st[4 + lane * kPerLane + e], U[e]);
  }

  const size_t bh = (size_t)b * a.H + h;
  if (nsplit == 1) {
    // the whole history was one chunk: finish here
    const float inv = (Lsum > 0.f) ? 1.f / Lsum : 0.f;
    __nv_bfloat16* out = a.o + bh * D + lane * kPerLane;
#pragma unroll
    for (int e = 0; e < kPerLane; e += 2)
      *reinterpret_cast<uint32_t*>(out + e) = pack_bf16x2(U[e] * inv, U[e + 1] * inv);
    if (lane == 0) a.lse[bh] = (Lsum > 0.f) ? (M + __log2f(Lsum)) * 0.69314718055994530942f : -INFINITY;
    return;
  }

  // write this CTA's state; the last CTA of (b, h) to finish merges them all
  {
    float* pu = a.part_u + (bh * a.splits + split) * D + lane * kPerLane;
    if constexpr (kPerLane == 4)
      __stcg(reinterpret_cast<float4*>(pu), make_float4(U[0], U[1], U[2], U[3]));
    else
      __stcg(reinterpret_cast<float2*>(pu), make_float2(U[0], U[1]));
    if (lane == 0) __stcg(reinterpret_cast<float2*>(a.part_ml) + bh * a.splits + split, make_float2(M, Lsum));
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
  const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + bh * a.splits;
  const float* pu = a.part_u + bh * a.splits * D + lane * kPerLane;
  M = -INFINITY;
  Lsum = 0.f;
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

DecodePlan decode_plan(int B, int H, int max_seqlen_k, int d, int num_splits, bool paged) {
  DecodePlan p;
  const int heads = paged ? DecLayout<128, false>::kHeads
                          : (d == 64 ? DecLayout<64, true>::kHeads : DecLayout<128, true>::kHeads);
  const int stage_keys = paged ? DecLayout<128, false>::kKeysPerStage
                               : (d == 64 ? DecLayout<64, true>::kKeysPerStage : DecLayout<128, true>::kKeysPerStage);
  static_assert(DecLayout<64, false>::kHeads == DecLayout<128, false>::kHeads &&
                    DecLayout<64, false>::kKeysPerStage == DecLayout<128, false>::kKeysPerStage,
                "the bulk-copy layout has the same head groups and stages for both d");
  p.heads_per_group = std::min(H, heads);
  p.groups = (H + heads - 1) / heads;
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
      // a small problem: spread it over one wave of CTAs (a CTA of a second wave
      // would start its first chunk only when one of the first wave retires)
      const long long units = (long long)B * p.groups;
      const long long s = std::max(1LL, slots / units);
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
  // chunks handed out: whole stages, about a sixteenth of a CTA's even share of the
  // keys and at most 256 keys, so the CTAs of a (sequence, group) can even out how
  // fast each is served: when the counter runs out, the CTAs still streaming hold at
  // most one chunk each (one request of 8192 keys, H = 32: chunks of one stage, 1
  // us faster than chunks of two)
  const int per = (chunk / 16 + stage_keys - 1) / stage_keys * stage_keys;
  p.gchunk = std::min(std::max(256, stage_keys), std::max(stage_keys, per));
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

template <int D, bool kTiled>
static fa_status launch_decode_impl(const DecodeLaunch& L0, cudaStream_t stream) {
  using L = DecLayout<D, kTiled>;
  static PerDeviceOnce attr_once;
  if (!attr_once.run([] {
        return cudaFuncSetAttribute(decode_kernel<D, kTiled>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::kSmemBytes) == cudaSuccess;
      }))
    return FA_ERR_CUDA;
  CUtensorMap tmK, tmV;
  memset(&tmK, 0, sizeof(tmK));
  memset(&tmV, 0, sizeof(tmV));
  if constexpr (kTiled) {
    // rows of the packed cache: the given count, else the most that B sequences of
    // at most max_seqlen_k keys can hold (the boxes never pass a sequence's end, so
    // this only bounds the map)
    const long long rows = L0.total_kv >= 0 ? (long long)L0.total_kv : (long long)L0.B * L0.max_seqlen_k;
    const int r = (int)std::max(1LL, std::min(rows, 0x7fffffffLL));
    if (!encode_rows_map(&tmK, L0.k, r, L0.H, D, L::kKeysPerStage) ||
        !encode_rows_map(&tmV, L0.v, r, L0.H, D, L::kKeysPerStage))
      return FA_ERR_CUDA;
  }
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
  const dim3 grid(L0.plan.groups, L0.plan.splits, L0.B);
  prof_before(stream, kKDecode);
  decode_kernel<D, kTiled><<<grid, kThreads, L::kSmemBytes, stream>>>(tmK, tmV, a);
  const cudaError_t err = cudaGetLastError();
  prof_after(stream, kKDecode);
  return err == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status launch_decode(const DecodeLaunch& L0, cudaStream_t stream) {
  const bool paged = L0.block_table != nullptr;
  if (L0.d == 64) return paged ? launch_decode_impl<64, false>(L0, stream) : launch_decode_impl<64, true>(L0, stream);
  if (L0.d == 128)
    return paged ? launch_decode_impl<128, false>(L0, stream) : launch_decode_impl<128, true>(L0, stream);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
