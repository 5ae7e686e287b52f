// sp_norm.cu — the sequence-parallel step around LayerNorm/Dropout (Megatron-style
// sequence parallelism), emulated on one GPU over N virtual tensor-parallel ranks.
//
// Page "序列并行：超长序列训练" (guijiagi.com), the MegatronSP example: after the
// tensor-parallel region a reduce-scatter along the sequence returns each rank its
// shard of the summed partial outputs; dropout is applied locally and the residual
// added; LayerNorm is per token and needs no communication. The 5688vip.com page's
// sequence_parallel_ln_dropout function fixes the LayerNorm (population variance,
// eps inside the square root, gamma * x_norm + beta) and training-mode dropout
// (kept values divided by 1 - rate). On one GPU the N ranks' shards are contiguous
// chunks of one [rows][H] buffer, so the all-gather of the shards is that buffer
// itself and the reduce-scatter is the sum of the N partials, chunk by chunk.
//
// One fused HBM pass per token row:
//   z = keep ? (sum_r partial_r) / (1 - p) : 0  (+ residual),   y = LayerNorm(z)
// The keep mask is an input (the random draw of dropout), one bit per element,
// bit i % 32 of word i / 32 for flat element i = row * H + h. z is kept in
// registers in fp32 between the two block reductions (mean, then the centred
// sum of squares), so the row is read once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sm100.cuh"
#include "sp_norm.h"

namespace cpattn {

namespace {

constexpr int kSpThreads = 128;
constexpr int kSpMaxVec = 8;   // 16-byte vectors per thread: H <= 128 * 8 * 8 = 8192

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();   // red[] of the previous reduction has been read
  if (lane == 0) red[warp] = v;
  __syncthreads();
  return (red[0] + red[1]) + (red[2] + red[3]);
}

__device__ __forceinline__ void unpack8(const uint4 u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(sm100::pack_bf16x2(f[0], f[1]), sm100::pack_bf16x2(f[2], f[3]),
                    sm100::pack_bf16x2(f[4], f[5]), sm100::pack_bf16x2(f[6], f[7]));
}

__global__ void __launch_bounds__(kSpThreads) sp_rs_dropout_add_ln_kernel(const SpArgs a) {
  __shared__ float red[4];
  const int nvec = a.H / 8;
  const float inv_h = 1.f / static_cast<float>(a.H);
  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    float v[kSpMaxVec][8];
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kSpMaxVec; ++j) {
      const int vi = threadIdx.x + kSpThreads * j;
      if (vi < nvec) {
        const int64_t e0 = row * a.H + static_cast<int64_t>(vi) * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int r = 0; r < a.nparts; ++r) {
          float f[8];
          unpack8(__ldg(reinterpret_cast<const uint4*>(a.partials + r * a.part_stride + e0)), f);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] += f[k];
        }
        if (a.keep != nullptr) {
          const uint32_t bits = (__ldg(a.keep + (e0 >> 5)) >> (e0 & 31)) & 0xffu;
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] = (bits >> k) & 1u ? acc[k] * a.inv_keep : 0.f;
        }
        if (a.residual != nullptr) {
          float f[8];
          unpack8(__ldg(reinterpret_cast<const uint4*>(a.residual + e0)), f);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] += f[k];
        }
        if (a.z != nullptr) *reinterpret_cast<uint4*>(a.z + e0) = pack8(acc);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          v[j][k] = acc[k];
          s += acc[k];
        }
      }
    }
    if (a.y == nullptr) continue;   // uniform across the block
    const float mean = block_sum(s, red) * inv_h;
    float q = 0.f;
#pragma unroll
    for (int j = 0; j < kSpMaxVec; ++j) {
      const int vi = threadIdx.x + kSpThreads * j;
      if (vi < nvec) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float d = v[j][k] - mean;
          q = fmaf(d, d, q);
        }
      }
    }
    const float rstd = rsqrtf(block_sum(q, red) * inv_h + a.eps);
#pragma unroll
    for (int j = 0; j < kSpMaxVec; ++j) {
      const int vi = threadIdx.x + kSpThreads * j;
      if (vi < nvec) {
        const int h0 = vi * 8;
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + h0));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + h0 + 4));
        const float4 b0 = __ldg(reinterpret_cast<const float4*>(a.beta + h0));
        const float4 b1 = __ldg(reinterpret_cast<const float4*>(a.beta + h0 + 4));
        const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        float o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = fmaf((v[j][k] - mean) * rstd, g[k], b[k]);
        *reinterpret_cast<uint4*>(a.y + row * a.H + h0) = pack8(o);
      }
    }
  }
}

}  // namespace

cudaError_t launch_sp_rs_dropout_add_ln(const SpArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = a.rows;
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  if (blocks > cap) blocks = cap;
  sp_rs_dropout_add_ln_kernel<<<static_cast<int>(blocks), kSpThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace cpattn
