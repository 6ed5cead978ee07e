// fa_abi.cu -- the C ABI of libfa.so: argument checks, workspace carving, TMA
// descriptor encoding and kernel launches.  No device memory is allocated here.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include <cmath>

#include "fa_internal.h"

namespace fa {

// ----------------------------------------------------------------------------- launch profiler

namespace {
const char* const kKernelNames[kKCount] = {"fa_fwd_kernel", "fa_bwd_preprocess_kernel", "fa_bwd_main_kernel",
                                           "fa_bwd_convert_kernel", "fa_decode_kernel",
                                           "fa_decode_check_kernel"};
struct ProfRecord {
  int kernel;
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};
std::vector<cudaEvent_t> g_event_pool;
size_t g_pool_used = 0;
std::vector<ProfRecord> g_records;
int g_launches[kKCount] = {};
double g_total_ms[kKCount] = {};
bool g_prof_error = false;

cudaEvent_t pool_event() {
  if (g_pool_used == g_event_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) {
      g_prof_error = true;
      return nullptr;
    }
    g_event_pool.push_back(e);
  }
  return g_event_pool[g_pool_used++];
}
}  // namespace

void prof_before(cudaStream_t s, int kernel_id) {
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  ProfRecord r;
  r.kernel = kernel_id;
  r.start = pool_event();
  r.stop = pool_event();
  if (!r.start || !r.stop) return;
  if (cudaEventRecord(r.start, s) != cudaSuccess) g_prof_error = true;
  g_records.push_back(r);
}

void prof_after(cudaStream_t s, int kernel_id) {
  if (!g_prof_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto it = g_records.rbegin(); it != g_records.rend(); ++it) {
    if (it->kernel == kernel_id) {
      if (cudaEventRecord(it->stop, s) != cudaSuccess) g_prof_error = true;
      return;
    }
  }
}

int num_sms() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    if (cached[dev] == 0) {
      int n = 0;
      if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
      cached[dev] = n;
    }
    return cached[dev];
  }
  return 148;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool encode_bshd_map(CUtensorMap* map, const void* ptr, int B, int N, int H, int D) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)N * H * D * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_rows_map(CUtensorMap* map, const void* ptr, int rows, int H, int D, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn || rows <= 0 || box_rows <= 0 || box_rows > 256) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

unsigned long long wait_timeout_ns() {
  static unsigned long long v = [] {
    unsigned long long ms = 2000;
    if (const char* env = getenv("FA_WAIT_TIMEOUT_MS")) {
      const unsigned long long x = strtoull(env, nullptr, 10);
      if (x > 0) ms = x;
    }
    return ms * 1000000ull;
  }();
  return v;
}

bool checks_enabled() {
  const char* env = getenv("FA_CHECKS");
  return env && env[0] == '1';
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

static bool dims_ok(int B, int H, int Nq, int Nk, int d) {
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0) return false;
  // TMA coordinates and the row arithmetic use 32-bit ints
  const long long rows_q = (long long)B * Nq * H, rows_k = (long long)B * Nk * H;
  return rows_q < (1LL << 31) && rows_k < (1LL << 31) && (long long)d * H < (1LL << 20);
}

static float resolve_scale(float s, int d) { return s > 0.f ? s : 1.0f / sqrtf((float)d); }

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_version(void) { return "0.1.0"; }

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
  }
  return "FA_ERR_UNKNOWN";
}

size_t fa_fwd_workspace_size(int B, int H, int Nq, int Nk, int d) {
  if (!dims_ok(B, H, Nq, Nk, d) || (d != 64 && d != 128)) return 0;
  return kStatusBytes;
}

size_t fa_bwd_workspace_size(int B, int H, int Nq, int Nk, int d) {
  if (!dims_ok(B, H, Nq, Nk, d) || (d != 64 && d != 128)) return 0;
  return kStatusBytes + up256(sizeof(float) * (size_t)B * Nq * H * d) + up256(sizeof(float) * (size_t)B * H * Nq);
}

size_t fa_bwd_varlen_workspace_size(int H, int total_q, int d) {
  // a packed batch is one batch element of total_q rows for the workspace arrays
  return fa_bwd_workspace_size(1, H, total_q, 1, d);
}

int fa_decode_num_splits(int B, int H, int max_seqlen_k, int d, int num_splits) {
  if (B <= 0 || H <= 0 || max_seqlen_k < 0 || (d != 64 && d != 128) || num_splits < 0) return 0;
  return decode_plan(B, H, max_seqlen_k, d, num_splits).splits;
}

size_t fa_decode_workspace_size(int B, int H, int max_seqlen_k, int d, int num_splits) {
  if (B <= 0 || H <= 0 || max_seqlen_k < 0 || (d != 64 && d != 128) || num_splits < 0) return 0;
  // one size serves the packed and the paged decode
  return std::max(decode_workspace_bytes(B, H, d, decode_plan(B, H, max_seqlen_k, d, num_splits, false)),
                  decode_workspace_bytes(B, H, d, decode_plan(B, H, max_seqlen_k, d, num_splits, true)));
}

// Dropout threshold t = round(65536 p) for 0 <= p < 1; false when p is out of range
// or so close to 1 that no draw would be kept.
static bool dropout_threshold(float p, uint32_t* t) {
  if (!(p >= 0.f && p < 1.f)) return false;
  const double x = std::floor((double)p * 65536.0 + 0.5);
  if (x >= 65536.0) return false;
  *t = (uint32_t)x;
  return true;
}

// Dense forward, with an optional key-padding mask (4-byte aligned when given),
// dropout (drop_t = 0: none) or block-sparse mask.
static fa_status fwd_dense(const void* q, const void* k, const void* v, void* o, float* lse, const uint32_t* key_mask,
                           uint32_t drop_t, unsigned long long seed, const uint8_t* block_mask, int causal_delta, int B,
                           int H, int Nq, int Nk, int d, int causal,
                           float softmax_scale, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse || !dims_ok(B, H, Nq, Nk, d)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(key_mask) & 3u))
    return FA_ERR_ALIGNMENT;
  if (!workspace || !aligned16(workspace) || workspace_bytes < fa_fwd_workspace_size(B, H, Nq, Nk, d))
    return FA_ERR_WORKSPACE;
  FwdLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.status = static_cast<int*>(workspace);
  a.key_mask = key_mask;
  a.drop_t = drop_t;
  a.seed = seed;
  a.block_mask = block_mask;
  a.causal_delta = causal_delta;
  a.B = B;
  a.H = H;
  a.Nq = Nq;
  a.Nk = Nk;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.scale = resolve_scale(softmax_scale, d);
  a.timeout_ns = wait_timeout_ns();
  return launch_fwd(a, stream);
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                 int d, int causal, float softmax_scale, void* workspace, size_t workspace_bytes,
                 cudaStream_t stream) {
  const NvtxRange range("fa_fwd");
  return fwd_dense(q, k, v, o, lse, nullptr, 0u, 0ull, nullptr, 0, B, H, Nq, Nk, d, causal, softmax_scale, workspace,
                   workspace_bytes, stream);
}

fa_status fa_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse, const uint32_t* key_mask,
                        float dropout_p, unsigned long long seed, int B, int H, int Nq, int Nk, int d, int causal,
                        float softmax_scale, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_fwd_masked");
  uint32_t t = 0;
  if (!dropout_threshold(dropout_p, &t)) return FA_ERR_INVALID_ARG;
  return fwd_dense(q, k, v, o, lse, key_mask, t, seed, nullptr, 0, B, H, Nq, Nk, d, causal, softmax_scale, workspace,
                   workspace_bytes, stream);
}

fa_status fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                             const uint8_t* block_mask, int B, int H, int Nq, int Nk, int d, int causal,
                             float softmax_scale, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_fwd_blocksparse");
  if (!block_mask) return FA_ERR_INVALID_ARG;
  return fwd_dense(q, k, v, o, lse, nullptr, 0u, 0ull, block_mask, 0, B, H, Nq, Nk, d, causal, softmax_scale, workspace,
                   workspace_bytes, stream);
}

// The shard holds keys key_offset .. key_offset + Nk - 1 of Nk_total: query i sees
// shard key j iff key_offset + j <= i + Nk_total - Nq, i.e. j <= i + (Nk - Nq) + delta
// with delta = Nk_total - key_offset - Nk.
static bool shard_delta(int key_offset, int Nk_total, int Nk, int* delta) {
  if (key_offset < 0 || Nk_total <= 0 || (long long)key_offset + Nk > Nk_total) return false;
  *delta = Nk_total - key_offset - Nk;
  return true;
}

fa_status fa_fwd_shard(const void* q, const void* k, const void* v, void* o, float* lse, int key_offset, int Nk_total,
                       int B, int H, int Nq, int Nk, int d, float softmax_scale, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_fwd_shard");
  int delta = 0;
  if (!shard_delta(key_offset, Nk_total, Nk, &delta)) return FA_ERR_INVALID_ARG;
  return fwd_dense(q, k, v, o, lse, nullptr, 0u, 0ull, nullptr, delta, B, H, Nq, Nk, d, 1, softmax_scale, workspace,
                   workspace_bytes, stream);
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                        const int32_t* cu_seqlens_k, void* o, float* lse, int B, int H, int total_q, int total_k,
                        int max_seqlen_q, int max_seqlen_k, int d, int causal, float softmax_scale, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_fwd_varlen");
  if (!q || !k || !v || !cu_seqlens_q || !cu_seqlens_k || !o || !lse) return FA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || total_q <= 0 || total_k <= 0 || max_seqlen_q <= 0 || max_seqlen_k <= 0)
    return FA_ERR_INVALID_ARG;
  if ((long long)total_q * H * d >= (1LL << 40) || (long long)total_k * H * d >= (1LL << 40) ||
      (long long)((max_seqlen_q + 255) / 256) * B * H >= (1LL << 31))
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return FA_ERR_ALIGNMENT;
  if (!workspace || !aligned16(workspace) || workspace_bytes < kStatusBytes) return FA_ERR_WORKSPACE;
  FwdLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.status = static_cast<int*>(workspace);
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.total_q = total_q;
  a.total_k = total_k;
  a.B = B;
  a.H = H;
  a.Nq = max_seqlen_q;
  a.Nk = max_seqlen_k;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.scale = resolve_scale(softmax_scale, d);
  a.timeout_ns = wait_timeout_ns();
  return launch_fwd(a, stream);
}

// Dense backward, with an optional key-padding mask (4-byte aligned when given),
// the forward's dropout (drop_t = 0: none) or block-sparse mask.
static fa_status bwd_dense(const void* q, const void* k, const void* v, const void* o, const void* do_,
                           const float* lse, void* dq, void* dk, void* dv, const uint32_t* key_mask, uint32_t drop_t,
                           unsigned long long seed, const uint8_t* block_mask, int causal_delta, int B, int H, int Nq,
                           int Nk, int d, int causal, float softmax_scale, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
  if (!q || !k || !v || !o || !do_ || !lse || !dq || !dk || !dv || !dims_ok(B, H, Nq, Nk, d))
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(do_) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(key_mask) & 3u))
    return FA_ERR_ALIGNMENT;
  if (!workspace || !aligned16(workspace) || workspace_bytes < fa_bwd_workspace_size(B, H, Nq, Nk, d))
    return FA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.dout = do_;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.status = reinterpret_cast<int*>(ws);
  a.dq_acc = reinterpret_cast<float*>(ws + kStatusBytes);
  a.delta = reinterpret_cast<float*>(ws + kStatusBytes + up256(sizeof(float) * (size_t)B * Nq * H * d));
  a.key_mask = key_mask;
  a.drop_t = drop_t;
  a.seed = seed;
  a.block_mask = block_mask;
  a.causal_delta = causal_delta;
  a.B = B;
  a.H = H;
  a.Nq = Nq;
  a.Nk = Nk;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.scale = resolve_scale(softmax_scale, d);
  a.timeout_ns = wait_timeout_ns();
  return launch_bwd(a, stream);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* do_, const float* lse,
                 void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int d, int causal,
                 float softmax_scale, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_bwd");
  return bwd_dense(q, k, v, o, do_, lse, dq, dk, dv, nullptr, 0u, 0ull, nullptr, 0, B, H, Nq, Nk, d, causal,
                   softmax_scale, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_masked(const void* q, const void* k, const void* v, const void* o, const void* do_,
                        const float* lse, void* dq, void* dk, void* dv, const uint32_t* key_mask, float dropout_p,
                        unsigned long long seed, int B, int H, int Nq, int Nk, int d, int causal,
                        float softmax_scale, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_bwd_masked");
  uint32_t t = 0;
  if (!dropout_threshold(dropout_p, &t)) return FA_ERR_INVALID_ARG;
  return bwd_dense(q, k, v, o, do_, lse, dq, dk, dv, key_mask, t, seed, nullptr, 0, B, H, Nq, Nk, d, causal,
                   softmax_scale, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const void* do_,
                             const float* lse, void* dq, void* dk, void* dv, const uint8_t* block_mask, int B, int H,
                             int Nq, int Nk, int d, int causal, float softmax_scale, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_bwd_blocksparse");
  if (!block_mask) return FA_ERR_INVALID_ARG;
  return bwd_dense(q, k, v, o, do_, lse, dq, dk, dv, nullptr, 0u, 0ull, block_mask, 0, B, H, Nq, Nk, d, causal,
                   softmax_scale, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_shard(const void* q, const void* k, const void* v, const void* o, const void* do_, const float* lse,
                       void* dq, void* dk, void* dv, int key_offset, int Nk_total, int B, int H, int Nq, int Nk, int d,
                       float softmax_scale, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_bwd_shard");
  int delta = 0;
  if (!shard_delta(key_offset, Nk_total, Nk, &delta)) return FA_ERR_INVALID_ARG;
  return bwd_dense(q, k, v, o, do_, lse, dq, dk, dv, nullptr, 0u, 0ull, nullptr, delta, B, H, Nq, Nk, d, 1,
                   softmax_scale, workspace, workspace_bytes, stream);
}

fa_status fa_merge_partials(const void* o_parts, const float* lse_parts, int S, int B, int H, int Nq, int d, void* o,
                            float* lse, cudaStream_t stream) {
  const NvtxRange range("fa_merge_partials");
  if (!o_parts || !lse_parts || !o || !lse || S <= 0 || !dims_ok(B, H, Nq, 1, d)) return FA_ERR_INVALID_ARG;
  if ((long long)S * B * Nq * H >= (1LL << 40)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(o_parts) || !aligned16(o) || !aligned16(lse_parts) || !aligned16(lse)) return FA_ERR_ALIGNMENT;
  return launch_merge(o_parts, lse_parts, S, B, H, Nq, d, o, lse, stream);
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* do_, const float* lse,
                        void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                        int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d, int causal,
                        float softmax_scale, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_bwd_varlen");
  if (!q || !k || !v || !o || !do_ || !lse || !dq || !dk || !dv || !cu_seqlens_q || !cu_seqlens_k)
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || max_seqlen_q <= 0 || max_seqlen_k <= 0 || !dims_ok(1, H, total_q, total_k, d))
    return FA_ERR_INVALID_ARG;
  // row coordinates of a tile (first row + up to 255) stay in 32 bits; the key-tile
  // grid fits one launch dimension
  if ((long long)total_q + 256 >= (1LL << 31) || (long long)total_k + 256 >= (1LL << 31) ||
      (long long)((max_seqlen_k + 127) / 128) * B * H >= (1LL << 31))
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(do_) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return FA_ERR_ALIGNMENT;
  if (!workspace || !aligned16(workspace) || workspace_bytes < fa_bwd_varlen_workspace_size(H, total_q, d))
    return FA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.dout = do_;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.status = reinterpret_cast<int*>(ws);
  a.dq_acc = reinterpret_cast<float*>(ws + kStatusBytes);
  a.delta = reinterpret_cast<float*>(ws + kStatusBytes + up256(sizeof(float) * (size_t)total_q * H * d));
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.total_q = total_q;
  a.total_k = total_k;
  a.B = B;
  a.H = H;
  a.Nq = max_seqlen_q;
  a.Nk = max_seqlen_k;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.scale = resolve_scale(softmax_scale, d);
  a.timeout_ns = wait_timeout_ns();
  return launch_bwd(a, stream);
}

}  // extern "C"

// The packed split-KV decode behind fa_decode_splitkv (total_kv = -1: offsets not
// checked against the buffers) and fa_decode_splitkv_checked.
static fa_status decode_packed(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_k, int B,
                               int H, int Nq, int total_kv, int max_seqlen_k, int d, float softmax_scale,
                               int num_splits, void* o, float* lse, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  if (!q || !k || !v || !cu_seqlens_k || !o || !lse) return FA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Nq != 1 || max_seqlen_k < 0 || num_splits < 0) return FA_ERR_INVALID_ARG;
  if ((long long)B * H >= (1LL << 31)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return FA_ERR_ALIGNMENT;
  const DecodePlan plan = decode_plan(B, H, max_seqlen_k, d, num_splits);
  if (!workspace || !aligned16(workspace) || workspace_bytes < decode_workspace_bytes(B, H, d, plan))
    return FA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.cu_seqlens = cu_seqlens_k;
  a.total_kv = total_kv;
  a.o = o;
  a.lse = lse;
  decode_carve(ws, B, H, d, plan, a);
  a.B = B;
  a.H = H;
  a.max_seqlen_k = max_seqlen_k;
  a.d = d;
  a.scale = resolve_scale(softmax_scale, d);
  a.plan = plan;
  a.check_args = checks_enabled() ? 1 : 0;
  a.timeout_ns = wait_timeout_ns();
  return launch_decode(a, stream);
}

extern "C" {

fa_status fa_decode_splitkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_k, int B, int H,
                            int Nq, int max_seqlen_k, int d, int causal, float softmax_scale, int num_splits, void* o,
                            float* lse, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_decode_splitkv");
  (void)causal;  // one query row: the bottom-right aligned mask admits every key
  return decode_packed(q, k, v, cu_seqlens_k, B, H, Nq, -1, max_seqlen_k, d, softmax_scale, num_splits, o, lse,
                       workspace, workspace_bytes, stream);
}

fa_status fa_decode_splitkv_checked(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_k,
                                    int B, int H, int Nq, int total_kv, int max_seqlen_k, int d, int causal,
                                    float softmax_scale, int num_splits, void* o, float* lse, void* workspace,
                                    size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_decode_splitkv_checked");
  (void)causal;
  if (total_kv < 0) return FA_ERR_INVALID_ARG;
  return decode_packed(q, k, v, cu_seqlens_k, B, H, Nq, total_kv, max_seqlen_k, d, softmax_scale, num_splits, o,
                       lse, workspace, workspace_bytes, stream);
}

fa_status fa_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                          const int32_t* seqlens_k, int B, int H, int num_pages, int page_size, int max_pages_per_seq,
                          int max_seqlen_k, int d, float softmax_scale, int num_splits, void* o, float* lse,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const NvtxRange range("fa_decode_paged");
  if (!q || !k_pages || !v_pages || !block_table || !seqlens_k || !o || !lse) return FA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || num_pages <= 0 || page_size <= 0 || max_pages_per_seq <= 0 || max_seqlen_k < 0 ||
      num_splits < 0)
    return FA_ERR_INVALID_ARG;
  if ((long long)B * H >= (1LL << 31) || (long long)B * max_pages_per_seq >= (1LL << 31)) return FA_ERR_INVALID_ARG;
  // every key a sequence may hold must have a block-table entry
  if ((long long)max_seqlen_k > (long long)max_pages_per_seq * page_size) return FA_ERR_INVALID_ARG;
  if ((long long)num_pages * page_size * H * (long long)d >= (1LL << 62)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seqlens_k) & 3u))
    return FA_ERR_ALIGNMENT;
  const DecodePlan plan = decode_plan(B, H, max_seqlen_k, d, num_splits, true);
  if (!workspace || !aligned16(workspace) || workspace_bytes < decode_workspace_bytes(B, H, d, plan))
    return FA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeLaunch a;
  a.q = q;
  a.k = k_pages;
  a.v = v_pages;
  a.cu_seqlens = nullptr;
  a.block_table = block_table;
  a.seqlens = seqlens_k;
  a.page_size = page_size;
  a.max_pages = max_pages_per_seq;
  a.num_pages = num_pages;
  a.o = o;
  a.lse = lse;
  decode_carve(ws, B, H, d, plan, a);
  a.B = B;
  a.H = H;
  a.max_seqlen_k = max_seqlen_k;
  a.d = d;
  a.scale = resolve_scale(softmax_scale, d);
  a.plan = plan;
  a.check_args = 0;
  a.timeout_ns = wait_timeout_ns();
  return launch_decode(a, stream);
}

fa_status fa_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_records.clear();
  g_pool_used = 0;
  g_prof_error = false;
  for (int i = 0; i < kKCount; ++i) {
    g_launches[i] = 0;
    g_total_ms[i] = 0.0;
  }
  g_prof_on.store(true);
  return FA_OK;
}

fa_status fa_profile_stop(void) {
  g_prof_on.store(false);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  bool bad = g_prof_error;
  for (const ProfRecord& r : g_records) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
      cudaGetLastError();
      bad = true;
      continue;
    }
    g_launches[r.kernel] += 1;
    g_total_ms[r.kernel] += ms;
  }
  g_records.clear();
  g_pool_used = 0;
  return bad ? FA_ERR_CUDA : FA_OK;
}

int fa_profile_count(void) { return kKCount; }

fa_status fa_profile_get(int id, const char** name, int* launches, double* total_ms) {
  if (id < 0 || id >= kKCount) return FA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (name) *name = kKernelNames[id];
  if (launches) *launches = g_launches[id];
  if (total_ms) *total_ms = g_total_ms[id];
  return FA_OK;
}

fa_status fa_check(void* workspace, cudaStream_t stream) {
  if (!workspace) return FA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  int status = 0;
  if (cudaMemcpy(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  if (status != 0) {
    const int zero = 0;
    if (cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
  }
  switch (status) {
    case 0: return FA_OK;
    case kStatusTimeout: return FA_ERR_TIMEOUT;
    case kStatusBadArg: return FA_ERR_INVALID_ARG;
    default: return FA_ERR_CUDA;
  }
}

}  // extern "C"
