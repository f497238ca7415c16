// rope.cu -- stand-alone in-place 3D RoPE of Q and K.
//
// Wan2.2 source reading, ch. 4, section "3D RoPE": per head, channels
// [0, 44) turn with the token's frame index f, [44, 86) with its row h and
// [86, 128) with its column w; adjacent channels (2j, 2j+1) form one complex
// number multiplied by exp(i * pos * theta^(-2j / D_band)).  The cos / sin
// come from the table wan_rope3d_table() writes (rows of 22 pairs: time,
// height with a trailing pad, width with a leading pad).
//
// HBM-bound: each 16-byte chunk (8 bf16 = 4 complex pairs) of Q / K is read
// and written once; the table (<= 70 KB) stays in L1 / L2.  One thread per
// chunk per trip, consecutive threads on consecutive chunks (coalesced),
// grid-stride over both tensors.
#include "wan_internal.cuh"

namespace wan {
namespace {

constexpr int kThreads = 256;

struct RopeArgs {
  uint4* q;
  uint4* k;
  const float4* table;  // rows of 11 float4 = 22 {cos, sin} pairs
  int64_t chunks;       // chunks per tensor = B * L * heads * 16
  int heads, F, H, W;
};

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
  float2 r;
  r.x = __uint_as_float(v << 16);
  r.y = __uint_as_float(v & 0xFFFF0000u);
  return r;
}

// Rotate the 4 complex pairs of one chunk.  `c` = chunk index in the head
// row (0..15): absolute pairs p = 4c .. 4c+3.  tt / th / tw point at the
// token's table rows (float4 = two pairs).
__device__ __forceinline__ uint4 rotate_chunk(uint4 raw, int c,
                                              const float4* tt,
                                              const float4* th,
                                              const float4* tw) {
  uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int p0 = 4 * c + 2 * half;  // even absolute pair index
    float4 cs;                        // {cos p0, sin p0, cos p0+1, sin p0+1}
    if (p0 + 1 < 22) {
      cs = tt[p0 >> 1];
    } else if (p0 >= 22 && p0 + 1 < 43) {
      cs = th[(p0 - 22) >> 1];
    } else if (p0 >= 44) {
      cs = tw[(p0 - 42) >> 1];
    } else {  // p0 = 42: pair 42 is the last height pair, 43 the first width
      const float4 a = th[10];  // entries 20, 21 -> pair 42 in .x/.y
      const float4 b = tw[0];   // entries 0 (pad), 1 -> pair 43 in .z/.w
      cs = make_float4(a.x, a.y, b.z, b.w);
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 v = bf16x2_to_float2(w[2 * half + e]);
      const float co = e ? cs.z : cs.x;
      const float si = e ? cs.w : cs.y;
      const float re = fmaf(v.x, co, -v.y * si);
      const float im = fmaf(v.x, si, v.y * co);
      w[2 * half + e] = pack_bf16x2(re, im);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(kThreads) rope3d_kernel(RopeArgs a) {
  const int64_t total = a.chunks * 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  const int hw = a.H * a.W;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
       g < total; g += stride) {
    const bool is_k = g >= a.chunks;
    const int64_t i = is_k ? g - a.chunks : g;
    uint4* base = is_k ? a.k : a.q;
    if (!base) continue;
    const int c = static_cast<int>(i & 15);
    const int64_t row = i >> 4;  // (b * L + n) * heads + head
    const int n = static_cast<int>((row / a.heads) % (static_cast<int64_t>(a.F) * hw));
    const int f = n / hw;
    const int h = (n / a.W) % a.H;
    const int w = n % a.W;
    const float4* tt = a.table + static_cast<int64_t>(f) * 11;
    const float4* th = a.table + static_cast<int64_t>(a.F + h) * 11;
    const float4* tw = a.table + static_cast<int64_t>(a.F + a.H + w) * 11;
    base[i] = rotate_chunk(base[i], c, tt, th, tw);
  }
}

}  // namespace
}  // namespace wan

extern "C" int wan_rope3d_qk(void* q, void* k, int B, wan_grid_t g,
                             int heads, int head_dim, const void* d_table,
                             void* s) {
  if (head_dim != 128 || B < 0 || heads < 1 || !d_table) return WAN_EINVAL;
  if (wan_rope3d_table_bytes(g, head_dim) == 0) return WAN_EINVAL;
  if ((!q && !k) || B == 0) return (B == 0 && (q || k)) ? WAN_OK : WAN_EINVAL;
  if ((q && !wan::aligned16(q)) || (k && !wan::aligned16(k)) ||
      !wan::aligned16(d_table))
    return WAN_EALIGN;
  if (q && q == k) return WAN_EINVAL;
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
  wan::RopeArgs a;
  a.q = static_cast<uint4*>(q);
  a.k = static_cast<uint4*>(k);
  a.table = static_cast<const float4*>(d_table);
  const int64_t L = static_cast<int64_t>(g.F) * g.H * g.W;
  a.chunks = static_cast<int64_t>(B) * L * heads * 16;
  a.heads = heads;
  a.F = g.F;
  a.H = g.H;
  a.W = g.W;
  int64_t blocks = (2 * a.chunks + wan::kThreads - 1) / wan::kThreads;
  const int64_t cap = static_cast<int64_t>(sm_count[dev]) * 8;
  if (blocks > cap) blocks = cap;
  wan::rope3d_kernel<<<static_cast<unsigned>(blocks), wan::kThreads, 0,
                       wan::as_stream(s)>>>(a);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}
