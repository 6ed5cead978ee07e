// decode_noalloc.cu -- split-KV decode for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device scratch memory: a plugin or custom
// operator whose host framework owns every device allocation and exposes no
// allocator, or a latency-critical serving loop that must never reach cudaMalloc
// (which can synchronise the device).  fa_decode_splitkv needs a caller-provided
// workspace for its per-chunk partial states; this variant instead keeps that
// scratch in a fixed array compiled into the library.  Its size is fixed at
// kNoAllocScratchBytes, and every GPU that loads the library holds that much
// memory until the process exits.
//
// The kernels and their launch are the ones of fa_decode_splitkv; only where the
// scratch comes from differs.
#include <mutex>

#include "fa_internal.h"

namespace fa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB

// The scratch itself.  In host code this name is only a host-side stand-in for
// the device symbol: its device address is looked up with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Device address of the scratch on the current device; looked up once per device
// and kept for the life of the process (a device reset after that is not
// supported: the kept address would no longer be valid).
fa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FA_OK;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" fa_status fa_decode_splitkv_noalloc(const void* q, const void* k, const void* v,
                                               const int32_t* cu_seqlens_k, int B, int H, int Nq,
                                               int max_seqlen_k, int d, int causal, float softmax_scale,
                                               int num_splits, void* o, float* lse, cudaStream_t stream) {
  const NvtxRange range("fa_decode_splitkv_noalloc");
  (void)causal;  // one query row: the bottom-right aligned mask admits every key
  if (!q || !k || !v || !cu_seqlens_k || !o || !lse) return FA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Nq != 1 || max_seqlen_k < 0 || num_splits < 0) return FA_ERR_INVALID_ARG;
  if ((long long)B * H >= (1LL << 31)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o) |
                        reinterpret_cast<uintptr_t>(lse);
  if ((mis & 15u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u)) return FA_ERR_ALIGNMENT;

  // scratch layout: status word | tickets [B*H] | chunk counters [B*H] | done counters
  // [B*H] | chunk (m, l) [B,H,S,2] | chunk u [B,H,S,d] (the counters need only B * groups
  // entries; B*H bounds that)
  const DecodePlan plan = decode_plan(B, H, max_seqlen_k, d, num_splits);
  const size_t off_tickets = kStatusBytes;
  const size_t off_ml = off_tickets + up256(sizeof(unsigned) * 3 * (size_t)B * H);
  const size_t off_u = off_ml + up256(sizeof(float) * 2 * (size_t)B * H * plan.splits);
  const size_t need = off_u + up256(sizeof(float) * (size_t)d * B * H * plan.splits);
  if (need > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;  // beyond the fixed scratch: pass fewer splits

  void* base = nullptr;
  const fa_status st = scratch_address(&base);
  if (st != FA_OK) return st;
  uint8_t* s = static_cast<uint8_t*>(base);
  // The array keeps whatever the previous call left: clear the status word, the
  // merge tickets and the chunk counters, which must start at zero.
  if (cudaMemsetAsync(s, 0, off_ml, stream) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }

  DecodeLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.cu_seqlens = cu_seqlens_k;
  a.o = o;
  a.lse = lse;
  a.status = reinterpret_cast<int*>(s);
  a.tickets = reinterpret_cast<unsigned*>(s + off_tickets);
  a.grab = a.tickets + (size_t)B * H;
  a.grab_done = a.grab + (size_t)B * H;
  a.clear_ptr = nullptr;  // cleared above together with the status word
  a.clear_bytes = 0;
  a.part_ml = reinterpret_cast<float*>(s + off_ml);
  a.part_u = reinterpret_cast<float*>(s + off_u);
  a.B = B;
  a.H = H;
  a.max_seqlen_k = max_seqlen_k;
  a.d = d;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)d);
  a.plan = plan;
  a.check_args = checks_enabled() ? 1 : 0;  // FA_CHECKS=1: cu_seqlens order checked first, as in fa_decode_splitkv
  a.timeout_ns = wait_timeout_ns();
  return launch_decode(a, stream);
}
