// merge_sm100.cu -- merging the partial results of attention over key shards.
//
// When the keys and values of a sequence are split into S shards (sequence
// parallelism across GPUs), attention over each shard gives a partial output o_s
// and log-sum-exp lse_s per query row.  They combine by the block-merge rule of
// "FlashAttention saves IO, not N^2 work", sections 3 and 7: with M = max_s lse_s,
//     O = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M),
//     lse = M + ln sum_s exp(lse_s - M).
// (o_s is already normalised by its shard's sum l_s = exp(lse_s - m_s), so the
// weights exp(lse_s - M) are the shards' l_s rescaled to the common reference.)
// A shard with lse_s = -inf (no visible key) contributes nothing; a row with no
// visible key in any shard gets O = 0 and lse = -inf.
//
// The kernel is HBM-bound: per row it reads S partial rows (bf16) and S lse values
// and writes one row.  D / 8 threads share a row, each owning 8 consecutive
// elements (one 16-byte load per shard).
#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {

namespace {

template <int D>
__global__ void __launch_bounds__(256) merge_partials_kernel(const uint4* __restrict__ o_parts,
                                                              const float* __restrict__ lse_parts,
                                                              uint4* __restrict__ o, float* __restrict__ lse, int S,
                                                              int B, int H, int Nq) {
  constexpr int kTpr = D / 8;  // threads per row
  const long long rows = (long long)B * Nq * H;
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / kTpr;
  const int part = threadIdx.x % kTpr;
  if (row >= rows) return;
  // row = (b * Nq + i) * H + h; lse is [B, H, Nq]
  const long long h = row % H, bi = row / H, bb = bi / Nq, i = bi % Nq;
  const long long lse_idx = (bb * H + h) * Nq + i;
  const long long lse_stride = (long long)B * H * Nq;  // between shards
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, __ldg(lse_parts + s * lse_stride + lse_idx));
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (M != -INFINITY) {
    const long long o_stride = rows * kTpr;  // uint4 per shard
    for (int s = 0; s < S; ++s) {
      const float ls = __ldg(lse_parts + s * lse_stride + lse_idx);
      if (ls == -INFINITY) continue;
      const float w = expf(ls - M);
      wsum += w;
      const uint4 x = __ldg(o_parts + s * o_stride + row * kTpr + part);
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] = fmaf(w, __uint_as_float(xs[e] << 16), acc[2 * e]);
        acc[2 * e + 1] = fmaf(w, __uint_as_float(xs[e] & 0xFFFF0000u), acc[2 * e + 1]);
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  o[row * kTpr + part] = make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                                    pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
  if (part == 0) lse[lse_idx] = wsum > 0.f ? M + logf(wsum) : -INFINITY;
}

template <int D>
fa_status launch_merge_impl(const void* o_parts, const float* lse_parts, int S, int B, int H, int Nq, void* o,
                            float* lse, cudaStream_t stream) {
  const long long threads = (long long)B * Nq * H * (D / 8);
  const long long grid = (threads + 255) / 256;
  if (grid > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  merge_partials_kernel<D><<<(unsigned)grid, 256, 0, stream>>>(static_cast<const uint4*>(o_parts), lse_parts,
                                                                 static_cast<uint4*>(o), lse, S, B, H, Nq);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

fa_status launch_merge(const void* o_parts, const float* lse_parts, int S, int B, int H, int Nq, int d, void* o,
                       float* lse, cudaStream_t stream) {
  if (d == 64) return launch_merge_impl<64>(o_parts, lse_parts, S, B, H, Nq, o, lse, stream);
  if (d == 128) return launch_merge_impl<128>(o_parts, lse_parts, S, B, H, Nq, o, lse, stream);
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
