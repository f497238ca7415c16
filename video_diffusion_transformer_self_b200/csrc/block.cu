// block.cu -- the memory-bound steps around the attention of one DiT block.
//
// Wan2.2 source reading, ch. 4, section "Full forward of one block": the
// self-attention input is norm1(x) * (1 + e[1]) + e[0] and the block output
// x + y * e[2], under fp32 autocast; section "3D RoPE": q and k each pass an
// RMSNorm (QK-Norm) after their linear layers and before the rotation.
//
//   wan_adaln_modulate  LayerNorm over the model dim (no affine, eps) then
//                       * (1 + scale[b]) + shift[b]; fp32 in, bf16 out (the
//                       input of the Q / K / V projections).
//   wan_qk_norm_rope    RMSNorm of q and k over all heads of a token with a
//                       per-channel weight, then the 3D RoPE, in place, bf16.
//   wan_gated_residual  x += y * gate[b]; x fp32, y bf16.
//
// All three are HBM-bound passes: one CTA or warp per token, 16-byte
// accesses, the token's row held in registers (modulate) or re-read from L2
// (QK-Norm), so each tensor crosses HBM once each way.
#include "wan_internal.cuh"

namespace wan {
namespace {

// ----------------------------------------------------- AdaLN modulate ----

constexpr int kModThreads = 128;
constexpr int kModMaxVec = 16;  // float4 per thread: D <= 128 * 4 * 16

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5;
  __syncthreads();  // red is reused by consecutive calls
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kModThreads / 32; ++w) t += red[w];
  return t;
}

// kVec float4 per thread (D <= 128 * 4 * kVec), picked from D so that the
// row's registers, and so the occupancy, follow the row length.
template <int kVec>
__global__ void __launch_bounds__(kModThreads)
    adaln_modulate_kernel(const float4* __restrict__ x,
                          const float4* __restrict__ shift,
                          const float4* __restrict__ scale,
                          uint2* __restrict__ out, int L, int D4, float eps) {
  __shared__ float red[kModThreads / 32];
  const int64_t tok = blockIdx.x;          // b * L + l
  const int b = static_cast<int>(tok / L);
  const float4* xr = x + tok * D4;
  float4 v[kVec];
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < kVec; ++u) {
    const int i = threadIdx.x + u * kModThreads;
    if (i < D4) {
      v[u] = xr[i];
      s += (v[u].x + v[u].y) + (v[u].z + v[u].w);
    }
  }
  const float inv_d = 1.0f / (4.0f * D4);
  const float mean = block_sum(s, red) * inv_d;
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < kVec; ++u) {
    const int i = threadIdx.x + u * kModThreads;
    if (i < D4) {
      const float a = v[u].x - mean, bb = v[u].y - mean;
      const float c = v[u].z - mean, d = v[u].w - mean;
      ss += (a * a + bb * bb) + (c * c + d * d);
    }
  }
  const float rstd = rsqrtf(block_sum(ss, red) * inv_d + eps);
  uint2* orow = out + tok * D4;
#pragma unroll
  for (int u = 0; u < kVec; ++u) {
    const int i = threadIdx.x + u * kModThreads;
    if (i < D4) {
      const float4 sh = __ldg(shift + static_cast<int64_t>(b) * D4 + i);
      const float4 sc = __ldg(scale + static_cast<int64_t>(b) * D4 + i);
      const float y0 = fmaf((v[u].x - mean) * rstd, 1.f + sc.x, sh.x);
      const float y1 = fmaf((v[u].y - mean) * rstd, 1.f + sc.y, sh.y);
      const float y2 = fmaf((v[u].z - mean) * rstd, 1.f + sc.z, sh.z);
      const float y3 = fmaf((v[u].w - mean) * rstd, 1.f + sc.w, sh.w);
      orow[i] = make_uint2(pack_bf16x2(y0, y1), pack_bf16x2(y2, y3));
    }
  }
}

// ------------------------------------------------------ QK-Norm + RoPE ----

constexpr int kNrThreads = 256;
constexpr int kNrWarps = kNrThreads / 32;

struct NormRopeArgs {
  uint4* t[2];            // q, k (either may be null)
  const float4* w[2];     // weights [heads * 128] per tensor
  const float4* table;    // RoPE rows of 11 float4
  int64_t tokens;
  int L, heads, F, H, W;
  float eps;
};

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
  float2 r;
  r.x = __uint_as_float(v << 16);
  r.y = __uint_as_float(v & 0xFFFF0000u);
  return r;
}

__device__ __forceinline__ float4 pair_cs(int p0, const float4* tt,
                                          const float4* th,
                                          const float4* tw) {
  if (p0 + 1 < 22) return __ldg(tt + (p0 >> 1));
  if (p0 >= 22 && p0 + 1 < 43) return __ldg(th + ((p0 - 22) >> 1));
  if (p0 >= 44) return __ldg(tw + ((p0 - 42) >> 1));
  const float4 lo = __ldg(th + 10);
  const float4 hi = __ldg(tw);
  return make_float4(lo.x, lo.y, hi.z, hi.w);
}

// (x * f * w_pair) rotated by {cos, sin}, packed to bf16x2.
__device__ __forceinline__ uint32_t norm_rot2(uint32_t v, float f, float w0,
                                              float w1, float co, float si) {
  const float2 x = bf16x2_to_float2(v);
  const float a = x.x * f * w0;
  const float b = x.y * f * w1;
  return pack_bf16x2(fmaf(a, co, -b * si), fmaf(a, si, b * co));
}

__global__ void __launch_bounds__(kNrThreads) qk_norm_rope_kernel(
    NormRopeArgs a) {
  const int lane = threadIdx.x & 31;
  const int c = lane & 15;      // 16-byte chunk of a head row
  const int hsub = lane >> 4;   // head parity of this half-warp
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * kNrWarps;
  const int hw = a.H * a.W;
  const float inv_dim = 1.0f / (128.0f * a.heads);
  for (int64_t tok = static_cast<int64_t>(blockIdx.x) * kNrWarps +
                     (threadIdx.x >> 5);
       tok < a.tokens; tok += wstride) {
    const int n = static_cast<int>(tok % a.L);
    const int f = n / hw;
    const int h = (n / a.W) % a.H;
    const int w = n % a.W;
    const float4* tt = a.table + static_cast<int64_t>(f) * 11;
    const float4* th = a.table + static_cast<int64_t>(a.F + h) * 11;
    const float4* tw = a.table + static_cast<int64_t>(a.F + a.H + w) * 11;
    const float4 cs0 = pair_cs(4 * c, tt, th, tw);
    const float4 cs1 = pair_cs(4 * c + 2, tt, th, tw);
    const int64_t row0 = tok * a.heads;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      uint4* t = a.t[which];
      if (!t) continue;
      // pass 1: sum of squares over all heads of this token
      float ss = 0.f;
#pragma unroll 4
      for (int hh = hsub; hh < a.heads; hh += 2) {
        const uint4 v = t[(row0 + hh) * 16 + c];
        const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = bf16x2_to_float2(vv[e]);
          ss = fmaf(x.x, x.x, fmaf(x.y, x.y, ss));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float fac = rsqrtf(ss * inv_dim + a.eps);
      // pass 2 (the row is re-read from L2): normalise, weight, rotate
      const float4* wt = a.w[which];
#pragma unroll 4
      for (int hh = hsub; hh < a.heads; hh += 2) {
        const int64_t idx = (row0 + hh) * 16 + c;
        const uint4 v = t[idx];
        const float4 w0 = __ldg(wt + hh * 32 + 2 * c);
        const float4 w1 = __ldg(wt + hh * 32 + 2 * c + 1);
        t[idx] = make_uint4(norm_rot2(v.x, fac, w0.x, w0.y, cs0.x, cs0.y),
                            norm_rot2(v.y, fac, w0.z, w0.w, cs0.z, cs0.w),
                            norm_rot2(v.z, fac, w1.x, w1.y, cs1.x, cs1.y),
                            norm_rot2(v.w, fac, w1.z, w1.w, cs1.z, cs1.w));
      }
    }
  }
}

// Register-resident variant for heads <= 2 * kRows (all Wan sizes: 12, 24
// and 40 heads).  One warp per (token, tensor) item: lane l holds chunk
// l & 15 of heads l >> 4, l >> 4 + 2, ... in registers, so the row is read
// from HBM once, in one batch of independent loads, and written once.  kRows
// is picked from the head count so that small rows keep a high occupancy.
constexpr int kNrMaxRows = 20;
constexpr int kNrRegThreads = 128;
constexpr int kNrRegWarps = kNrRegThreads / 32;

// resident CTAs per SM that each row-register budget allows
template <int kRows>
constexpr int nr_min_blocks() {
  return kRows <= 4 ? 8 : kRows <= 12 ? 6 : 3;
}

template <int kRows>
__global__ void __launch_bounds__(kNrRegThreads, nr_min_blocks<kRows>())
    qk_norm_rope_reg_kernel(NormRopeArgs a) {
  const int lane = threadIdx.x & 31;
  const int c = lane & 15;
  const int hsub = lane >> 4;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * kNrRegWarps;
  const int hw = a.H * a.W;
  const float inv_dim = 1.0f / (128.0f * a.heads);
  // items: (token, tensor) with the present tensors interleaved per token
  const int ntens = (a.t[0] != nullptr) + (a.t[1] != nullptr);
  const int first = a.t[0] != nullptr ? 0 : 1;
  const int64_t items = a.tokens * ntens;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * kNrRegWarps +
                    (threadIdx.x >> 5);
       it < items; it += wstride) {
    const int64_t tok = ntens == 2 ? (it >> 1) : it;
    const int which = ntens == 2 ? static_cast<int>(it & 1) : first;
    // select, not index: a runtime index into the parameter arrays would
    // copy them to the stack
    uint4* t = which ? a.t[1] : a.t[0];
    const int64_t row0 = tok * a.heads;
    uint4 r[kRows];
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      const int hh = hsub + 2 * k;
      if (hh < a.heads) r[k] = t[(row0 + hh) * 16 + c];
    }
    const int n = static_cast<int>(tok % a.L);
    const int f = n / hw;
    const int h = (n / a.W) % a.H;
    const int w = n % a.W;
    const float4* tt = a.table + static_cast<int64_t>(f) * 11;
    const float4* th = a.table + static_cast<int64_t>(a.F + h) * 11;
    const float4* tw = a.table + static_cast<int64_t>(a.F + a.H + w) * 11;
    const float4 cs0 = pair_cs(4 * c, tt, th, tw);
    const float4 cs1 = pair_cs(4 * c + 2, tt, th, tw);
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      if (hsub + 2 * k < a.heads) {
        const uint32_t vv[4] = {r[k].x, r[k].y, r[k].z, r[k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = bf16x2_to_float2(vv[e]);
          ss = fmaf(x.x, x.x, fmaf(x.y, x.y, ss));
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float fac = rsqrtf(ss * inv_dim + a.eps);
    const float4* wt = which ? a.w[1] : a.w[0];
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      const int hh = hsub + 2 * k;
      if (hh < a.heads) {
        const float4 w0 = __ldg(wt + hh * 32 + 2 * c);
        const float4 w1 = __ldg(wt + hh * 32 + 2 * c + 1);
        t[(row0 + hh) * 16 + c] =
            make_uint4(norm_rot2(r[k].x, fac, w0.x, w0.y, cs0.x, cs0.y),
                       norm_rot2(r[k].y, fac, w0.z, w0.w, cs0.z, cs0.w),
                       norm_rot2(r[k].z, fac, w1.x, w1.y, cs1.x, cs1.y),
                       norm_rot2(r[k].w, fac, w1.z, w1.w, cs1.z, cs1.w));
      }
    }
  }
}

// ---------------------------------------------------- gated residual ----

constexpr int kResThreads = 256;

__global__ void __launch_bounds__(kResThreads)
    gated_residual_kernel(float4* __restrict__ x, const uint2* __restrict__ y,
                          const float4* __restrict__ gate, int64_t n4,
                          int64_t per_batch4, int D4) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kResThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kResThreads +
                   threadIdx.x;
       i < n4; i += stride) {
    const int64_t b = i / per_batch4;
    const int d = static_cast<int>(i % D4);
    const float4 g = __ldg(gate + b * D4 + d);
    const uint2 yy = y[i];
    const float2 y01 = bf16x2_to_float2(yy.x);
    const float2 y23 = bf16x2_to_float2(yy.y);
    float4 xv = x[i];
    xv.x = fmaf(y01.x, g.x, xv.x);
    xv.y = fmaf(y01.y, g.y, xv.y);
    xv.z = fmaf(y23.x, g.z, xv.z);
    xv.w = fmaf(y23.y, g.w, xv.w);
    x[i] = xv;
  }
}

int sm_count_of(int dev) {
  static int sm[64];
  if (dev < 0 || dev >= 64) return 0;
  if (sm[dev] == 0) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) !=
        cudaSuccess)
      return 0;
    sm[dev] = c;
  }
  return sm[dev];
}

}  // namespace
}  // namespace wan

extern "C" {

int wan_adaln_modulate(const float* x, const float* shift, const float* scale,
                       void* out, int B, int L, int D, float eps, void* s) {
  if (!x || !shift || !scale || !out || B < 1 || L < 1 || D < 4 ||
      D % 4 != 0 || D > wan::kModThreads * 4 * wan::kModMaxVec ||
      !(eps > 0.f))
    return WAN_EINVAL;
  if (static_cast<int64_t>(B) * L > (1ll << 31) - 1) return WAN_EINVAL;
  if (!wan::aligned16(x) || !wan::aligned16(shift) || !wan::aligned16(scale) ||
      !wan::aligned16(out))
    return WAN_EALIGN;
  int st = wan::check_device(nullptr);
  if (st != WAN_OK) return st;
  const int D4 = D / 4;
  const int vec = (D4 + wan::kModThreads - 1) / wan::kModThreads;
  const unsigned nb = static_cast<unsigned>(B * L);
  cudaStream_t st_ = wan::as_stream(s);
  const float4* x4 = reinterpret_cast<const float4*>(x);
  const float4* sh4 = reinterpret_cast<const float4*>(shift);
  const float4* sc4 = reinterpret_cast<const float4*>(scale);
  uint2* o2 = static_cast<uint2*>(out);
  if (vec <= 3)
    wan::adaln_modulate_kernel<3><<<nb, wan::kModThreads, 0, st_>>>(
        x4, sh4, sc4, o2, L, D4, eps);
  else if (vec <= 6)
    wan::adaln_modulate_kernel<6><<<nb, wan::kModThreads, 0, st_>>>(
        x4, sh4, sc4, o2, L, D4, eps);
  else if (vec <= 10)
    wan::adaln_modulate_kernel<10><<<nb, wan::kModThreads, 0, st_>>>(
        x4, sh4, sc4, o2, L, D4, eps);
  else
    wan::adaln_modulate_kernel<wan::kModMaxVec>
        <<<nb, wan::kModThreads, 0, st_>>>(x4, sh4, sc4, o2, L, D4, eps);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}

int wan_qk_norm_rope(void* q, void* k, const float* wq, const float* wk,
                     int B, wan_grid_t g, int heads, int head_dim,
                     const void* d_table, float eps, void* s) {
  if (head_dim != 128 || B < 1 || heads < 1 || !d_table || !(eps > 0.f))
    return WAN_EINVAL;
  if (wan_rope3d_table_bytes(g, head_dim) == 0) return WAN_EINVAL;
  if (!q && !k) return WAN_EINVAL;
  if ((q && !wq) || (k && !wk)) return WAN_EINVAL;
  if ((q && (!wan::aligned16(q) || !wan::aligned16(wq))) ||
      (k && (!wan::aligned16(k) || !wan::aligned16(wk))) ||
      !wan::aligned16(d_table))
    return WAN_EALIGN;
  if (q && q == k) return WAN_EINVAL;
  int dev = 0;
  int st = wan::check_device(&dev);
  if (st != WAN_OK) return st;
  wan::NormRopeArgs a;
  a.t[0] = static_cast<uint4*>(q);
  a.t[1] = static_cast<uint4*>(k);
  a.w[0] = reinterpret_cast<const float4*>(wq);
  a.w[1] = reinterpret_cast<const float4*>(wk);
  a.table = static_cast<const float4*>(d_table);
  a.L = g.F * g.H * g.W;
  a.tokens = static_cast<int64_t>(B) * a.L;
  a.heads = heads;
  a.F = g.F;
  a.H = g.H;
  a.W = g.W;
  a.eps = eps;
  const bool reg = heads <= 2 * wan::kNrMaxRows;
  const int64_t items = reg ? a.tokens * ((q != nullptr) + (k != nullptr))
                            : a.tokens;
  const int wpb = reg ? wan::kNrRegWarps : wan::kNrWarps;
  // the variant for this head count (rows of 8 heads' uint4 per lane)
  const void* kern =
      !reg          ? reinterpret_cast<const void*>(wan::qk_norm_rope_kernel)
      : heads <= 8  ? reinterpret_cast<const void*>(
                          wan::qk_norm_rope_reg_kernel<4>)
      : heads <= 16 ? reinterpret_cast<const void*>(
                          wan::qk_norm_rope_reg_kernel<8>)
      : heads <= 24 ? reinterpret_cast<const void*>(
                          wan::qk_norm_rope_reg_kernel<12>)
                    : reinterpret_cast<const void*>(
                          wan::qk_norm_rope_reg_kernel<wan::kNrMaxRows>);
  // Measured at 32,760 tokens x 12 heads: the 8-per-SM cap launched 1,184
  // CTAs of which 888 fit, and the 1.33 waves ran at 4.5 TB/s; the grid of
  // resident CTAs runs at 5.6 TB/s (40 heads: +2 %).  The plain streaming
  // passes (RoPE, Euler and UniPC steps, transpose) measured 1-4 % faster
  // with their larger grids and keep them.
  int64_t blocks = (items + wpb - 1) / wpb;
  const int64_t cap = wan::resident_grid(
      kern, reg ? wan::kNrRegThreads : wan::kNrThreads, dev);
  if (cap < 1) return WAN_ECUDA;
  if (blocks > cap) blocks = cap;
  const unsigned nb = static_cast<unsigned>(blocks);
  cudaStream_t st_ = wan::as_stream(s);
  if (reg && heads <= 8)
    wan::qk_norm_rope_reg_kernel<4><<<nb, wan::kNrRegThreads, 0, st_>>>(a);
  else if (reg && heads <= 16)
    wan::qk_norm_rope_reg_kernel<8><<<nb, wan::kNrRegThreads, 0, st_>>>(a);
  else if (reg && heads <= 24)
    wan::qk_norm_rope_reg_kernel<12><<<nb, wan::kNrRegThreads, 0, st_>>>(a);
  else if (reg)
    wan::qk_norm_rope_reg_kernel<wan::kNrMaxRows>
        <<<nb, wan::kNrRegThreads, 0, st_>>>(a);
  else
    wan::qk_norm_rope_kernel<<<nb, wan::kNrThreads, 0, st_>>>(a);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}

int wan_gated_residual(float* x, const void* y, const float* gate, int B,
                       int L, int D, void* s) {
  if (!x || !y || !gate || B < 1 || L < 1 || D < 4 || D % 4 != 0)
    return WAN_EINVAL;
  if (!wan::aligned16(x) || !wan::aligned16(gate) ||
      (reinterpret_cast<uintptr_t>(y) & 7u) != 0)
    return WAN_EALIGN;
  int dev = 0;
  int st = wan::check_device(&dev);
  if (st != WAN_OK) return st;
  const int64_t per_batch4 = static_cast<int64_t>(L) * (D / 4);
  const int64_t n4 = per_batch4 * B;
  int64_t blocks = (n4 + wan::kResThreads - 1) / wan::kResThreads;
  const int64_t cap = static_cast<int64_t>(wan::sm_count_of(dev)) * 8;
  if (cap > 0 && blocks > cap) blocks = cap;
  wan::gated_residual_kernel<<<static_cast<unsigned>(blocks),
                               wan::kResThreads, 0, wan::as_stream(s)>>>(
      reinterpret_cast<float4*>(x), static_cast<const uint2*>(y),
      reinterpret_cast<const float4*>(gate), n4, per_batch4, D / 4);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}

}  // extern "C"
