// unipc.cu -- fused UniPC (order 2) sampler step: CFG combine, clean-sample
// estimate, corrector of the step just taken and predictor of the next one,
// in one pass over the latent.
//
// Wan2.2 source reading, ch. 5 "UniPC": the default integrator predicts the
// next stop from the trend of the last two model outputs and, once the model
// has been evaluated there, corrects the step just taken with that output at
// no extra forward.  Ch. 1 "From DDPM to flow matching": x = (1 - sigma) x0 +
// sigma noise and the clean estimate is x - sigma v.  The pages give no
// coefficients; they come from the published UniPC order conditions (Zhao et
// al., 2023) in data-prediction form, solved exactly:
//   lambda = log((1 - sigma) / sigma),  h = lambda_t - lambda_s,
//   q_k(h) = k! / h^k * integral_0^h exp(tau - h) tau^k / k! dtau,
//   x_t = (sigma_t / sigma_s) x_s
//         + (1 - sigma_t) (q_0 m_s + sum_j c_j (m_j - m_s) / r_j),
//   sum_j c_j r_j^(k-1) = q_k(h) for k = 1 .. #differences,
// r_j = (lambda_j - lambda_s) / h: r < 0 for an earlier stop, r = 1 for the
// new one (corrector).  Order 2 predictor unless no earlier stop at finite
// lambda exists or the target is sigma = 0 (first order there); the
// corrector uses the predictor's differences plus the new point.
//
// Per element (fp32, coefficients folded on the host in fp64):
//   v  = has_uncond ? fma(w, c - u, u) : c
//   m  = x - sigma v                                        -> m_out
//   xc = i == 0 ? x : cx xc + cm1 m1 + cm2 m2 + cm m        -> x_corr
//   x  = px xc + pm m + pm1 m1                              -> x
// HBM-bound: 36 bytes per element with CFG and the order-2 corrector (six
// fp32 reads, three writes).
#include <math.h>

#include "wan_internal.cuh"

namespace wan {

namespace {

// q_k(h) above: the alternating series k! sum_n (-1)^n h^(n+1) / (n+k+1)!
// for h <= 1, the recurrence q_k = 1 - k q_(k-1) / h (integration by parts)
// from q_0 = 1 - exp(-h) above that, and 1 at h = +inf.
double q_fn(int k, double h) {
  if (isinf(h)) return 1.0;
  if (h <= 1.0) {
    double t = h / (k + 1), sum = 0.0;
    for (int n = 0; n < 30; ++n) {
      sum += t;
      t *= -h / (n + k + 2);
    }
    return sum;
  }
  double q = -expm1(-h);
  for (int j = 1; j <= k; ++j) q = 1.0 - j * q / h;
  return q;
}

double lam(double s) {
  if (s <= 0.0) return INFINITY;
  if (s >= 1.0) return -INFINITY;
  return log((1.0 - s) / s);
}

// Order of the predictor from stop i to stop i + 1.
int pred_order(const double* sg, int i) {
  return (i >= 1 && sg[i + 1] > 0.0 && sg[i - 1] < 1.0) ? 2 : 1;
}

__device__ __forceinline__ float4 ld_stream(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 "
               "{%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

struct Coef {
  float sigma, w;
  float cx, cm1, cm2, cm;
  float px, pm, pm1;
};

// kMode 0: no corrector (first stop); 1: corrector on the new point only;
// 2: corrector with the earlier difference too (reads m_(i-2)).
template <bool kCfg, int kMode>
__device__ __forceinline__ void step1(float x, float c, float u, float xc,
                                      float m1, float m2, const Coef& k,
                                      float& x_out, float& xc_out,
                                      float& m_out) {
  const float v = kCfg ? fmaf(k.w, c - u, u) : c;
  const float m = fmaf(-k.sigma, v, x);
  float xn;
  if (kMode == 0) {
    xn = x;
  } else {
    xn = fmaf(k.cm, m, fmaf(k.cm1, m1, k.cx * xc));
    if (kMode == 2) xn = fmaf(k.cm2, m2, xn);
  }
  float y = fmaf(k.pm, m, k.px * xn);
  if (kMode != 0) y = fmaf(k.pm1, m1, y);
  x_out = y;
  xc_out = xn;
  m_out = m;
}

constexpr int kThreads = 256;
constexpr int kUnroll = 2;

template <bool kCfg, int kMode>
__global__ void __launch_bounds__(kThreads)
    unipc_kernel(float* __restrict__ x, float* __restrict__ xc,
                 const float* __restrict__ m1, const float* m2, float* m_out,
                 const float* __restrict__ vc, const float* __restrict__ vu,
                 const Coef k, int64_t n) {
  const int64_t n4 = n >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  float4* x4 = reinterpret_cast<float4*>(x);
  float4* xc4 = reinterpret_cast<float4*>(xc);
  float4* mo4 = reinterpret_cast<float4*>(m_out);
  const float4* m14 = reinterpret_cast<const float4*>(m1);
  const float4* m24 = reinterpret_cast<const float4*>(m2);
  const float4* c4 = reinterpret_cast<const float4*>(vc);
  const float4* u4 = reinterpret_cast<const float4*>(vu);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (; i < n4; i += kUnroll * stride) {
    float4 a[kUnroll], c[kUnroll], u[kUnroll], p[kUnroll], q1[kUnroll],
        q2[kUnroll];
    // All loads of the trip first (m_out may alias m2: each element is read
    // before the same thread writes it).
#pragma unroll
    for (int r = 0; r < kUnroll; ++r) {
      const int64_t j = i + r * stride;
      if (j < n4) {
        // x, x_corr and m_(i-2) are written by this kernel: plain loads;
        // the read-only inputs bypass L1.
        a[r] = x4[j];
        c[r] = ld_stream(c4 + j);
        u[r] = kCfg ? ld_stream(u4 + j) : z;
        p[r] = kMode ? xc4[j] : z;
        q1[r] = kMode ? ld_stream(m14 + j) : z;
        q2[r] = kMode == 2 ? m24[j] : z;
      }
    }
#pragma unroll
    for (int r = 0; r < kUnroll; ++r) {
      const int64_t j = i + r * stride;
      if (j < n4) {
        float4 ox, oc, om;
        step1<kCfg, kMode>(a[r].x, c[r].x, u[r].x, p[r].x, q1[r].x, q2[r].x,
                           k, ox.x, oc.x, om.x);
        step1<kCfg, kMode>(a[r].y, c[r].y, u[r].y, p[r].y, q1[r].y, q2[r].y,
                           k, ox.y, oc.y, om.y);
        step1<kCfg, kMode>(a[r].z, c[r].z, u[r].z, p[r].z, q1[r].z, q2[r].z,
                           k, ox.z, oc.z, om.z);
        step1<kCfg, kMode>(a[r].w, c[r].w, u[r].w, p[r].w, q1[r].w, q2[r].w,
                           k, ox.w, oc.w, om.w);
        x4[j] = ox;
        xc4[j] = oc;
        mo4[j] = om;
      }
    }
  }
  // Ragged tail of n % 4 elements.
  if (blockIdx.x == 0 && threadIdx.x < (n & 3)) {
    const int64_t j = (n4 << 2) + threadIdx.x;
    float ox, oc, om;
    step1<kCfg, kMode>(x[j], vc[j], kCfg ? vu[j] : 0.f, kMode ? xc[j] : 0.f,
                       kMode ? m1[j] : 0.f, kMode == 2 ? m2[j] : 0.f, k, ox,
                       oc, om);
    x[j] = ox;
    xc[j] = oc;
    m_out[j] = om;
  }
}

template <bool kCfg>
void launch(int mode, unsigned blocks, cudaStream_t s, float* x, float* xc,
            const float* m1, const float* m2, float* mo, const float* vc,
            const float* vu, const Coef& k, int64_t n) {
  if (mode == 0)
    unipc_kernel<kCfg, 0><<<blocks, kThreads, 0, s>>>(x, xc, m1, m2, mo, vc,
                                                       vu, k, n);
  else if (mode == 1)
    unipc_kernel<kCfg, 1><<<blocks, kThreads, 0, s>>>(x, xc, m1, m2, mo, vc,
                                                       vu, k, n);
  else
    unipc_kernel<kCfg, 2><<<blocks, kThreads, 0, s>>>(x, xc, m1, m2, mo, vc,
                                                       vu, k, n);
}

}  // namespace
}  // namespace wan

extern "C" int wan_unipc_coeffs(const double* sigmas, int n_steps, int i,
                                wan_unipc_coef_t* out) {
  if (!sigmas || !out || n_steps < 1 || i < 0 || i >= n_steps)
    return WAN_EINVAL;
  for (int j = 0; j <= n_steps; ++j) {
    const double s = sigmas[j];
    if (!(s >= 0.0 && s <= 1.0)) return WAN_EINVAL;  // NaN fails too
    if (j < n_steps && !(s > 0.0 && s > sigmas[j + 1])) return WAN_EINVAL;
  }
  using wan::lam;
  using wan::q_fn;
  const double* sg = sigmas;
  wan_unipc_coef_t c = {};
  c.sigma = sg[i];
  // Predictor from stop i (corrected sample) to stop i + 1.
  {
    const double h = lam(sg[i + 1]) - lam(sg[i]);
    const double a = sg[i + 1] / sg[i], al = 1.0 - sg[i + 1];
    c.pred_order = wan::pred_order(sg, i);
    c.px = a;
    if (c.pred_order == 2) {
      const double r = (lam(sg[i - 1]) - lam(sg[i])) / h;
      const double k1 = q_fn(1, h) / r;  // on (m_(i-1) - m_i)
      c.pm = al * (q_fn(0, h) - k1);
      c.pm1 = al * k1;
    } else {
      c.pm = al * q_fn(0, h);
      c.pm1 = 0.0;
    }
  }
  // Corrector of the step from stop i - 1 to stop i.
  if (i >= 1) {
    const double h = lam(sg[i]) - lam(sg[i - 1]);
    const double a = sg[i] / sg[i - 1], al = 1.0 - sg[i];
    const double q0 = q_fn(0, h), q1 = q_fn(1, h);
    c.cx = a;
    if (wan::pred_order(sg, i - 1) == 2) {
      // [1 1; r1 1] [c1; cn] = [q1; q2]
      const double r1 = (lam(sg[i - 2]) - lam(sg[i - 1])) / h;
      const double q2 = q_fn(2, h);
      const double c1 = (q1 - q2) / (1.0 - r1), cn = q1 - c1;
      c.corr_order = 2;
      c.cm2 = al * c1 / r1;
      c.cm = al * cn;
      c.cm1 = al * (q0 - c1 / r1 - cn);
    } else {
      c.corr_order = 1;
      c.cm = al * q1;
      c.cm1 = al * (q0 - q1);
      c.cm2 = 0.0;
    }
  }
  *out = c;
  return WAN_OK;
}

extern "C" int wan_unipc_step(float* x, float* x_corr, const float* m_prev1,
                              const float* m_prev2, float* m_out,
                              const float* v_cond, const float* v_uncond,
                              float guide, int64_t n, const double* sigmas,
                              int n_steps, int i, void* s) {
  wan_unipc_coef_t cf;
  int st = wan_unipc_coeffs(sigmas, n_steps, i, &cf);
  if (st != WAN_OK) return st;
  if (n < 0 || !isfinite(guide)) return WAN_EINVAL;
  if (n == 0) return WAN_OK;
  const int mode = cf.corr_order;  // 0, 1 or 2
  if (!x || !x_corr || !m_out || !v_cond) return WAN_EINVAL;
  if (mode >= 1 && !m_prev1) return WAN_EINVAL;
  if (mode == 2 && !m_prev2) return WAN_EINVAL;
  const void* used[6] = {x, x_corr, m_out, v_cond, v_uncond,
                         mode >= 1 ? m_prev1 : nullptr};
  for (int a = 0; a < 6; ++a) {
    if (used[a] && !wan::aligned16(used[a])) return WAN_EALIGN;
    for (int b = a + 1; b < 6; ++b)
      if (used[a] && used[a] == used[b]) return WAN_EINVAL;
  }
  if (mode == 2) {
    if (!wan::aligned16(m_prev2)) return WAN_EALIGN;
    // m_out may alias m_prev2 only
    for (int a = 0; a < 6; ++a)
      if (a != 2 && used[a] == m_prev2) return WAN_EINVAL;
  }
  int dev = 0;
  st = wan::check_device(&dev);
  if (st != WAN_OK) return st;
  static int sm_count[64];
  if (sm_count[dev] == 0) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) !=
        cudaSuccess)
      return WAN_ECUDA;
    sm_count[dev] = c;
  }
  wan::Coef k;
  k.sigma = static_cast<float>(cf.sigma);
  k.w = guide;
  k.cx = static_cast<float>(cf.cx);
  k.cm1 = static_cast<float>(cf.cm1);
  k.cm2 = static_cast<float>(cf.cm2);
  k.cm = static_cast<float>(cf.cm);
  k.px = static_cast<float>(cf.px);
  k.pm = static_cast<float>(cf.pm);
  k.pm1 = static_cast<float>(cf.pm1);
  const int64_t n4 = n >> 2;
  int64_t blocks = (n4 + wan::kThreads - 1) / wan::kThreads;
  const int64_t cap = static_cast<int64_t>(sm_count[dev]) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  cudaStream_t stream = wan::as_stream(s);
  if (v_uncond)
    wan::launch<true>(mode, static_cast<unsigned>(blocks), stream, x, x_corr,
                      m_prev1, m_prev2, m_out, v_cond, v_uncond, k, n);
  else
    wan::launch<false>(mode, static_cast<unsigned>(blocks), stream, x, x_corr,
                       m_prev1, m_prev2, m_out, v_cond, nullptr, k, n);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}
