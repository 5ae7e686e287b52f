// merge_permute.cu — the HBM-bound kernels: the merge of (O, lse) partials and
// the layout permutations (zigzag / contiguous rank-major, Ulysses head groups),
// plus the bounded-wait self-test kernel.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_fwd.h"
#include "sm100.cuh"

namespace cpattn {

namespace {

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// ------------------------------------------------------------------ merge
// Page "序列与上下文并行", section "上下文并行：注意力本身切分": the per-step partial
// results are merged by online softmax. Per row: M = max_t lse_t,
// lse = M + ln sum_t exp(lse_t - M), O = sum_t exp(lse_t - lse) O_t. A partial
// with lse_t = -inf has weight 0 and its O_t is not read; a row whose partials
// are all -inf gets O = 0, lse = -inf.
//
// D/4 threads per row, one float4 of O_t per thread per part: a warp reads
// 512 contiguous bytes per part and row pair, so every access is coalesced.
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(int P, int64_t rows, const float* __restrict__ o_parts,
                                                    const float* __restrict__ lse_parts,
                                                    __nv_bfloat16* __restrict__ o_out,
                                                    float* __restrict__ lse_out) {
  constexpr int kTpr = D / 4;         // threads per row
  constexpr int kRpw = 32 / kTpr;     // rows per warp
  const int lane = threadIdx.x & 31;
  const int sub = lane / kTpr;
  const int c = lane % kTpr;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = warp0 * kRpw; base < rows; base += nwarps * kRpw) {
    const int64_t r = base + sub;
    if (r >= rows) continue;
    float M = -INFINITY;
    for (int t = 0; t < P; ++t) M = fmaxf(M, __ldg(lse_parts + t * rows + r));
    const float Ms = M == -INFINITY ? 0.f : M;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float tot = 0.f;
#pragma unroll 4
    for (int t = 0; t < P; ++t) {
      const float w = expf(__ldg(lse_parts + t * rows + r) - Ms);   // 0 for an empty part
      if (w != 0.f) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(o_parts + (t * rows + r) * D) + c);
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
        tot += w;
      }
    }
    const float inv = tot > 0.f ? 1.f / tot : 0.f;
    uint2 out;
    out.x = sm100::pack_bf16x2(acc.x * inv, acc.y * inv);
    out.y = sm100::pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(o_out + r * D)[c] = out;
    if (lse_out != nullptr && c == 0) lse_out[r] = M == -INFINITY ? -INFINITY : Ms + logf(tot);
  }
}

// ------------------------------------------------------------------ permutations
// Source unit (token row or head-group run) of output unit `o`.
//   kind 0, dir 0: rank-major row o = (r*B + b)*T + tl <- natural row b*S + pos(r, tl)
//   kind 0, dir 1: natural row o = b*S + s <- rank-major row of token s
//   kind 1, dir 0: group run o = (g*B + b)*S + s <- shard run ((rho*B + b)*Sl + sl)*N + g
//   kind 1, dir 1: shard run o = ((rho*B + b)*Sl + sl)*N + g <- group run (g*B + b)*S + rho*Sl + sl
struct UnitMap {
  int kind, dir, N, B, S, zigzag;
  __device__ __forceinline__ int64_t src(int64_t o) const {
    if (kind == 0) {
      const int T = S / N;
      if (dir == 0) {
        const int tl = static_cast<int>(o % T);
        const int64_t rbv = o / T;
        const int b = static_cast<int>(rbv % B);
        const int r = static_cast<int>(rbv / B);
        int64_t pos;
        if (!zigzag) {
          pos = static_cast<int64_t>(r) * T + tl;
        } else {
          const int C = T / 2;
          pos = tl < C ? static_cast<int64_t>(r) * C + tl : static_cast<int64_t>(2 * N - 1 - r) * C + (tl - C);
        }
        return static_cast<int64_t>(b) * S + pos;
      }
      const int s = static_cast<int>(o % S);
      const int b = static_cast<int>(o / S);
      int r, tl;
      if (!zigzag) {
        r = s / T;
        tl = s % T;
      } else {
        const int C = T / 2;
        const int k = s / C;
        if (k < N) {
          r = k;
          tl = s % C;
        } else {
          r = 2 * N - 1 - k;
          tl = C + s % C;
        }
      }
      return (static_cast<int64_t>(r) * B + b) * T + tl;
    }
    const int Sl = S / N;
    if (dir == 0) {
      const int s = static_cast<int>(o % S);
      const int64_t gb = o / S;
      const int b = static_cast<int>(gb % B);
      const int g = static_cast<int>(gb / B);
      const int rho = s / Sl, sl = s % Sl;
      return ((static_cast<int64_t>(rho) * B + b) * Sl + sl) * N + g;
    }
    const int g = static_cast<int>(o % N);
    const int64_t rest = o / N;
    const int sl = static_cast<int>(rest % Sl);
    const int64_t rb = rest / Sl;
    const int b = static_cast<int>(rb % B);
    const int rho = static_cast<int>(rb / B);
    return (static_cast<int64_t>(g) * B + b) * S + static_cast<int64_t>(rho) * Sl + sl;
  }
};

// One warp per unit; each lane moves 16-byte vectors with a 512-byte stride.
__global__ void __launch_bounds__(256) permute_kernel(UnitMap m, int64_t units, int vec_per_unit,
                                                      const uint4* __restrict__ in, uint4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t u = warp0; u < units; u += nwarps) {
    const int64_t s = m.src(u);
    const uint4* src = in + s * vec_per_unit;
    uint4* dst = out + u * vec_per_unit;
    int v = lane;
    for (; v + 96 < vec_per_unit; v += 128) {
      const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64), d = __ldg(src + v + 96);
      dst[v] = a;
      dst[v + 32] = b;
      dst[v + 64] = c;
      dst[v + 96] = d;
    }
    for (; v < vec_per_unit; v += 32) dst[v] = __ldg(src + v);
  }
}

// Rotary position embedding fused into the forward gather (natural or Ulysses
// shards -> the attention view). Page "序列与上下文并行" (ai-infra-wiki), section
// "工程实践": under CP the position encoding of a token is computed at its GLOBAL
// position. Feature pair (2i, 2i+1) of every head at global position p is
// rotated by p * theta_i, theta_i = base^(-2i/D) (the frequencies of the pages'
// sinusoidal PositionalEncoding). The global position of an output unit is its
// natural token index (source row mod S for token rows; output run mod S for
// Ulysses head-group runs) plus pos_offset.
//
// The angle and its reduction to [-pi, pi] are computed in fp64 (positions up to
// 2^31 keep full fp32 accuracy of the reduced angle), then sincosf. A warp's 32
// lanes x 8 bf16 span whole heads (D in {64, 128}), so every lane always holds
// the same four feature pairs: it takes their cos/sin once per unit and applies
// them to all its 16-byte vectors.
__global__ void __launch_bounds__(256) rope_permute_kernel(UnitMap m, int64_t units, int vec_per_unit, RopeArgs ra,
                                                           const uint4* __restrict__ in, uint4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int i0 = ((8 * lane) % ra.D) / 2;   // first feature pair of this lane's vectors
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
  for (int64_t u = warp0; u < units; u += nwarps) {
    const int64_t s = m.src(u);
    const int64_t p = (m.kind == 0 ? s % m.S : u % m.S) + ra.pos_offset;
    float c[4], sn[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const double a = static_cast<double>(p) * ra.theta[i0 + k];
      const double r = a - rint(a * kInvTwoPi) * kTwoPi;
      sincosf(static_cast<float>(r), &sn[k], &c[k]);
    }
    const uint4* src = in + s * vec_per_unit;
    uint4* dst = out + u * vec_per_unit;
    for (int v = lane; v < vec_per_unit; v += 32) {
      const uint4 x = __ldg(src + v);
      uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float xe = __uint_as_float(w[k] << 16);          // feature 2i
        const float xo = __uint_as_float(w[k] & 0xffff0000u);  // feature 2i+1
        w[k] = sm100::pack_bf16x2(xe * c[k] - xo * sn[k], xe * sn[k] + xo * c[k]);
      }
      dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

__global__ void index_map_kernel(UnitMap m, int64_t units, int64_t* __restrict__ map) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < units; i += stride)
    map[i] = m.src(i);
}

// ------------------------------------------------------------------ wait probe
// One thread waits, with the same bounded wait the attention kernel uses, on a
// barrier that nothing arrives on; the wait runs out and records the timeout.
__global__ void wait_probe_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ sm100::WaitBlock wblk;
  if (threadIdx.x == 0) {
    sm100::mbar_init(sm100::smem_addr(&bar), 1);
    const sm100::WaitCtl ctl = sm100::wait_block_init(wblk, status, limit_ns);
    sm100::fence_barrier_init();
    sm100::mbar_wait(sm100::smem_addr(&bar), 0, ctl);
  }
}

UnitMap make_map(const PermuteArgs& a) {
  UnitMap m;
  m.kind = a.kind;
  m.dir = a.direction;
  m.N = a.N;
  m.B = a.B;
  m.S = a.S;
  m.zigzag = a.zigzag;
  return m;
}

}  // namespace

cudaError_t launch_merge(int num_parts, int64_t rows, int D, const float* o_parts, const float* lse_parts,
                         __nv_bfloat16* o_out, float* lse_out, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int rpw = 32 / (D / 4);
  const int64_t warps = (rows + rpw - 1) / rpw;
  int64_t blocks = (warps + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  if (D == 128)
    merge_kernel<128><<<static_cast<int>(blocks), 256, 0, stream>>>(num_parts, rows, o_parts, lse_parts, o_out, lse_out);
  else
    merge_kernel<64><<<static_cast<int>(blocks), 256, 0, stream>>>(num_parts, rows, o_parts, lse_parts, o_out, lse_out);
  return cudaGetLastError();
}

cudaError_t launch_permute(const PermuteArgs& a, const void* in, void* out, cudaStream_t stream) {
  const int64_t total_bytes = static_cast<int64_t>(a.B) * a.S * a.H * a.D * a.elem_bytes;
  const int64_t units = a.kind == 0 ? static_cast<int64_t>(a.B) * a.S : static_cast<int64_t>(a.N) * a.B * a.S;
  if (units == 0) return cudaSuccess;
  const int64_t unit_bytes = total_bytes / units;
  const int vpu = static_cast<int>(unit_bytes / 16);
  int64_t blocks = (units + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  permute_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(make_map(a), units, vpu,
                                                               static_cast<const uint4*>(in), static_cast<uint4*>(out));
  return cudaGetLastError();
}

cudaError_t launch_rope_permute(const PermuteArgs& a, const RopeArgs& ra, const void* in, void* out,
                                cudaStream_t stream) {
  const int64_t units = a.kind == 0 ? static_cast<int64_t>(a.B) * a.S : static_cast<int64_t>(a.N) * a.B * a.S;
  if (units == 0) return cudaSuccess;
  const int64_t unit_elems = (static_cast<int64_t>(a.B) * a.S * a.H * a.D) / units;
  const int vpu = static_cast<int>(unit_elems / 8);   // 16-byte vectors of bf16
  int64_t blocks = (units + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  rope_permute_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
      make_map(a), units, vpu, ra, static_cast<const uint4*>(in), static_cast<uint4*>(out));
  return cudaGetLastError();
}

cudaError_t launch_index_map(const PermuteArgs& a, int64_t* map_out, cudaStream_t stream) {
  PermuteArgs f = a;
  f.direction = 0;
  const int64_t units = a.kind == 0 ? static_cast<int64_t>(a.B) * a.S : static_cast<int64_t>(a.N) * a.B * a.S;
  if (units == 0) return cudaSuccess;
  int64_t blocks = (units + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  index_map_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(make_map(f), units, map_out);
  return cudaGetLastError();
}

cudaError_t launch_wait_probe(int* status, uint64_t limit_ns, cudaStream_t stream) {
  wait_probe_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace cpattn
