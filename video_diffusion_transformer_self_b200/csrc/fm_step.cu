// fm_step.cu -- fused classifier-free-guidance combine + Euler flow step.
//
// Wan2.2 source reading, ch. 5: Euler holds the velocity constant over the
// step (x <- x - dsigma * v, sigma decreasing) and CFG forms
// uncond + w * (cond - uncond).  Per element, in fp32:
//   v = has_uncond ? fma(w, c - u, u) : c
//   x = fma(dt, v, x)            with dt = sigma_next - sigma
// HBM-bound: 12 bytes per element (x read + written, v read), 16 with CFG.
// Vectorised 16-byte accesses, velocities streamed past L1/L2 residency,
// grid-stride over whole-SM-count multiples, 4 float4 per thread per trip.
#include "wan_internal.cuh"

namespace wan {

namespace {

__device__ __forceinline__ float4 ld_stream(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 "
               "{%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

template <bool kCfg>
__device__ __forceinline__ float4 step4(float4 x, float4 c, float4 u,
                                        float w, float dt) {
  if (kCfg) {
    c.x = fmaf(w, c.x - u.x, u.x);
    c.y = fmaf(w, c.y - u.y, u.y);
    c.z = fmaf(w, c.z - u.z, u.z);
    c.w = fmaf(w, c.w - u.w, u.w);
  }
  x.x = fmaf(dt, c.x, x.x);
  x.y = fmaf(dt, c.y, x.y);
  x.z = fmaf(dt, c.z, x.z);
  x.w = fmaf(dt, c.w, x.w);
  return x;
}

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

template <bool kCfg>
__global__ void __launch_bounds__(kThreads)
    fm_step_kernel(float* __restrict__ x, const float* __restrict__ vc,
                   const float* __restrict__ vu, float w, float dt,
                   int64_t n) {
  float4* x4 = reinterpret_cast<float4*>(x);
  const float4* c4 = reinterpret_cast<const float4*>(vc);
  const float4* u4 = reinterpret_cast<const float4*>(vu);
  const int64_t n4 = n >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  // Main body: kUnroll independent float4 triples in flight per thread.
  for (; i + (kUnroll - 1) * stride < n4; i += kUnroll * stride) {
    float4 xv[kUnroll], cv[kUnroll], uv[kUnroll];
#pragma unroll
    for (int r = 0; r < kUnroll; ++r) {
      xv[r] = x4[i + r * stride];
      cv[r] = ld_stream(c4 + i + r * stride);
      if (kCfg) uv[r] = ld_stream(u4 + i + r * stride);
    }
#pragma unroll
    for (int r = 0; r < kUnroll; ++r)
      x4[i + r * stride] = step4<kCfg>(xv[r], cv[r], uv[r], w, dt);
  }
  for (; i < n4; i += stride) {
    float4 uv = make_float4(0.f, 0.f, 0.f, 0.f);
    if (kCfg) uv = ld_stream(u4 + i);
    x4[i] = step4<kCfg>(x4[i], ld_stream(c4 + i), uv, w, dt);
  }
  // Ragged tail of n % 4 elements.
  if (blockIdx.x == 0 && threadIdx.x < (n & 3)) {
    const int64_t j = (n4 << 2) + threadIdx.x;
    float v = vc[j];
    if (kCfg) v = fmaf(w, v - vu[j], vu[j]);
    x[j] = fmaf(dt, v, x[j]);
  }
}

}  // namespace
}  // namespace wan

extern "C" int wan_fm_step(float* x, const float* v_cond,
                           const float* v_uncond, float guide, int64_t n,
                           double sigma, double sigma_next, void* s) {
  if (n < 0 || (n > 0 && (!x || !v_cond))) return WAN_EINVAL;
  if (!isfinite(sigma) || !isfinite(sigma_next) || !isfinite(guide))
    return WAN_EINVAL;
  if (n == 0) return WAN_OK;
  if (!wan::aligned16(x) || !wan::aligned16(v_cond) ||
      (v_uncond && !wan::aligned16(v_uncond)))
    return WAN_EALIGN;
  if (x == v_cond || x == v_uncond) return WAN_EINVAL;
  int dev = 0;
  int st = wan::check_device(&dev);
  if (st != WAN_OK) return st;
  static int sm_count[64];
  if (sm_count[dev] == 0) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) !=
        cudaSuccess)
      return WAN_ECUDA;
    sm_count[dev] = c;
  }
  const float dt = static_cast<float>(sigma_next - sigma);
  const int64_t n4 = n >> 2;
  // 8 resident 256-thread blocks per SM; fewer for small problems.
  int64_t blocks = (n4 + wan::kThreads - 1) / wan::kThreads;
  const int64_t cap = static_cast<int64_t>(sm_count[dev]) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  cudaStream_t stream = wan::as_stream(s);
  if (v_uncond)
    wan::fm_step_kernel<true><<<static_cast<unsigned>(blocks), wan::kThreads,
                                0, stream>>>(x, v_cond, v_uncond, guide, dt, n);
  else
    wan::fm_step_kernel<false><<<static_cast<unsigned>(blocks),
                                 wan::kThreads, 0, stream>>>(
        x, v_cond, nullptr, guide, dt, n);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}
