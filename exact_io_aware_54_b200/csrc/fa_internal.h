// fa_internal.h -- declarations shared by the C ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include <nvtx3/nvToolsExt.h>  // header-only NVTX v3: a range costs a pointer check unless a profiler listens

#include "fa.h"  // include/ (on the compiler include path)

namespace fa {

// An NVTX range named after the entry point, open for the duration of the call,
// so that a profiler's timeline shows which library call launched which kernels.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Workspace: the first kStatusBytes hold the status word (int32) and padding; the
// forward's item counters use bytes 128 .. 135 of the padding (zero between calls).
constexpr size_t kStatusBytes = 256;

// Decode counters live in a fixed region right after the status word, so they
// stay at the same place whatever the shape of the call: the merge tickets of
// every (sequence, head), then the key-chunk counters and the done-counters of
// every (sequence, head group).  Each resets itself at the end of a call (the
// last merge of a (sequence, head) clears its ticket, the last producer of a
// (sequence, group) its two counters).  Calls with more than kDecodeFixedTickets
// (sequence, head) pairs use a region after the partial states that is cleared
// on every call.
constexpr size_t kDecodeFixedTickets = 65536;
constexpr size_t kDecodeSyncBytes = 3 * kDecodeFixedTickets * 4;

// Status codes recorded by kernels in the workspace status word (fa_status values).
constexpr int kStatusTimeout = 6;
constexpr int kStatusBadArg = 1;

// Kernels the library launches (for the optional launch profiler).
enum KernelId { kKFwd = 0, kKBwdPre, kKBwdMain, kKBwdConvert, kKDecode, kKDecodeCheck, kKCount };
// Bracket a launch with profiling events when profiling is on (no-ops otherwise).
void prof_before(cudaStream_t s, int kernel_id);
void prof_after(cudaStream_t s, int kernel_id);

// Number of SMs of the current device (cached per device).
int num_sms();

// Wall-time limit of every bounded wait inside a kernel: FA_WAIT_TIMEOUT_MS
// milliseconds when set (and positive), else 2 s.  Read once per process.
unsigned long long wait_timeout_ns();

// FA_CHECKS=1 turns on the optional device-side argument checks.
bool checks_enabled();

// One-time, per-device set-up (a kernel attribute, say) that is safe when several
// host threads make their first call at the same time: the first caller on a
// device runs `set` under a lock, the others wait for it; after a success later
// calls only read an atomic flag.  A failed `set` is retried by the next call.
class PerDeviceOnce {
 public:
  template <class F>
  bool run(F&& set) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    if (dev < 0 || dev >= kMaxDevices) return set();  // outside the table: set up on every call
    if (done_[dev].load(std::memory_order_acquire)) return true;
    std::lock_guard<std::mutex> lk(mu_);
    if (done_[dev].load(std::memory_order_relaxed)) return true;
    if (!set()) return false;
    done_[dev].store(true, std::memory_order_release);
    return true;
  }

 private:
  static constexpr int kMaxDevices = 64;
  std::atomic<bool> done_[kMaxDevices]{};
  std::mutex mu_;
};

// Encode a TMA descriptor for a bf16 tensor [B, N, H, D] (D innermost), with a
// box of 128 rows x 64 columns and 128-byte swizzle.  Returns false on failure.
bool encode_bshd_map(CUtensorMap* map, const void* ptr, int B, int N, int H, int D);
// Map of a packed [rows, H, D] bf16 tensor with boxes of 64 columns x one head x
// box_rows rows, 128-byte swizzled (zeros outside the tensor).
bool encode_rows_map(CUtensorMap* map, const void* ptr, int rows, int H, int D, int box_rows);

// The same for an fp32 tensor [B, N, H, D]: box of 128 rows x 32 columns (128 bytes), 128-byte swizzle.

struct FwdLaunch {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int* status;
  // variable-length batch (cu_q != nullptr): q, o are [total_q, H, d], k, v
  // [total_k, H, d], lse [H, total_q]; Nq, Nk are the maximum sequence lengths
  const int32_t* cu_q = nullptr;
  const int32_t* cu_k = nullptr;
  int total_q = 0, total_k = 0;
  // key-padding mask (dense batches): device uint32 [B, ceil(Nk / 32)], bit j % 32
  // of word j / 32 set when key j takes part; null for none
  const uint32_t* key_mask = nullptr;
  // dropout: drop_t = round(65536 p) (0: none), seed of the Philox draws
  uint32_t drop_t = 0;
  unsigned long long seed = 0;
  // block-sparse mask (dense batches): device uint8 [H, ceil(Nq/128), ceil(Nk/128)],
  // 0 skips the (query tile, KV tile) block; null for dense attention
  const uint8_t* block_mask = nullptr;
  // causal visibility offset beyond the bottom-right alignment (a key shard: its
  // keys start later in the sequence)
  int causal_delta = 0;
  int B, H, Nq, Nk, d, causal;
  float scale;
  unsigned long long timeout_ns;
};
fa_status launch_fwd(const FwdLaunch& a, cudaStream_t stream);

struct BwdLaunch {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* dq_acc;  // [B, Nq, H, d] fp32 ([total_q, H, d] when packed)
  float* delta;   // [B, H, Nq] fp32 ([H, total_q] when packed)
  int* status;
  // variable-length batch (cu_q != nullptr): q, o, dout, dq are [total_q, H, d],
  // k, v, dk, dv [total_k, H, d], lse [H, total_q]; Nq, Nk are the maximum lengths
  const int32_t* cu_q = nullptr;
  const int32_t* cu_k = nullptr;
  int total_q = 0, total_k = 0;
  const uint32_t* key_mask = nullptr;  // as for the forward
  uint32_t drop_t = 0;                  // as for the forward
  unsigned long long seed = 0;
  const uint8_t* block_mask = nullptr;  // as for the forward
  int causal_delta = 0;                 // as for the forward
  int B, H, Nq, Nk, d, causal;
  float scale;
  unsigned long long timeout_ns;
};
fa_status launch_bwd(const BwdLaunch& a, cudaStream_t stream);

// Merge of S partial (o, lse) results over key shards (merge_sm100.cu).
fa_status launch_merge(const void* o_parts, const float* lse_parts, int S, int B, int H, int Nq, int d, void* o,
                       float* lse, cudaStream_t stream);

// Split-KV decode plan: keys per chunk and chunks per sequence.
struct DecodePlan {
  int chunk;       // keys per CTA if the keys were split evenly (multiple of 8)
  int splits;      // CTAs (and partial states) per (sequence, head group)
  int gchunk;      // keys per chunk handed out to a CTA (whole stages of the decode ring)
  int groups;      // head groups per sequence
  int heads_per_group;
};
// paged: the plan of the paged-cache kernel (other head groups and stages)
DecodePlan decode_plan(int B, int H, int max_seqlen_k, int d, int num_splits, bool paged = false);

struct DecodeLaunch {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* cu_seqlens;  // packed cache: [B + 1] row offsets (nullptr when paged)
  // paged cache (block_table != nullptr): k, v are [num_pages, page_size, H, d];
  // key t of sequence b is row t % page_size of page block_table[b * max_pages + t / page_size]
  const int32_t* block_table = nullptr;
  const int32_t* seqlens = nullptr;  // [B] keys per sequence
  int page_size = 0, max_pages = 0, num_pages = 0;
  void* o;
  float* lse;
  int* status;
  unsigned int* tickets;    // [B * H] merge tickets, zero between calls
  unsigned int* grab;       // [B * groups] key-chunk counters, zero between calls
  unsigned int* grab_done;  // [B * groups] producers done, zero between calls
  void* clear_ptr = nullptr;  // counters outside the fixed region: cleared before the launch
  size_t clear_bytes = 0;
  float* part_ml;      // [B, H, splits, 2]  (m in log2 units, l)
  float* part_u;       // [B, H, splits, d]
  int B, H, max_seqlen_k, d;
  float scale;
  DecodePlan plan;
  int check_args;      // validate cu_seqlens on the device first
  // packed cache: rows in k and v (>= 0: a sequence whose rows do not lie in
  // [0, total_kv) is skipped and recorded as a bad argument; -1: not checked)
  int total_kv = -1;
  unsigned long long timeout_ns;
};
fa_status launch_decode(const DecodeLaunch& a, cudaStream_t stream);

size_t decode_workspace_bytes(int B, int H, int d, const DecodePlan& plan);

// Points the status word, counters and partial states of `a` into a caller
// workspace of at least decode_workspace_bytes(B, H, d, plan) bytes.
void decode_carve(uint8_t* ws, int B, int H, int d, const DecodePlan& plan, DecodeLaunch& a);

}  // namespace fa
