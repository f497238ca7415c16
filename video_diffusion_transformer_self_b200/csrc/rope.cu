// rope.cu -- stand-alone in-place 3D RoPE of Q and K.
//
// Wan2.2 source reading, ch. 4, section "3D RoPE": per head, channels
// [0, 44) turn with the token's frame index f, [44, 86) with its row h and
// [86, 128) with its column w; adjacent channels (2j, 2j+1) form one complex
// number multiplied by exp(i * pos * theta^(-2j / D_band)).  The cos / sin
// come from the table wan_rope3d_table() writes (rows of 22 pairs: time,
// height with a trailing pad, width with a leading pad).
//
// HBM-bound: every 16-byte chunk (8 bf16 = 4 complex pairs) of Q / K is read
// and written once.  One warp per token (grid-stride over B * L tokens): the
// token's (f, h, w) is found once, lane l owns chunk c = l & 15 of every
// head row, loads the 4 cos / sin pairs of that chunk once, and walks the
// heads two at a time (lanes 0-15 head 2i, lanes 16-31 head 2i+1), so each
// warp access covers 512 contiguous bytes.
#include "wan_internal.cuh"

namespace wan {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 4;  // head rows per lane per batch

struct RopeArgs {
  uint4* q;
  uint4* k;
  const float4* table;  // rows of 11 float4 = 22 {cos, sin} pairs
  int64_t tokens;       // B * L
  int L, heads, F, H, W;
};

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
  float2 r;
  r.x = __uint_as_float(v << 16);
  r.y = __uint_as_float(v & 0xFFFF0000u);
  return r;
}

// {cos, sin} of absolute pairs p0 and p0 + 1 (p0 even) for the token whose
// band rows are tt (time), th (height), tw (width).
__device__ __forceinline__ float4 pair_cs(int p0, const float4* tt,
                                          const float4* th,
                                          const float4* tw) {
  if (p0 + 1 < 22) return __ldg(tt + (p0 >> 1));
  if (p0 >= 22 && p0 + 1 < 43) return __ldg(th + ((p0 - 22) >> 1));
  if (p0 >= 44) return __ldg(tw + ((p0 - 42) >> 1));
  // p0 = 42: pair 42 is the last height pair, pair 43 the first width pair
  const float4 lo = __ldg(th + 10);  // entries 20, 21 -> pair 42 in .x/.y
  const float4 hi = __ldg(tw);       // entries 0 (pad), 1 -> pair 43 in .z/.w
  return make_float4(lo.x, lo.y, hi.z, hi.w);
}

__device__ __forceinline__ uint32_t rot2(uint32_t v, float co, float si) {
  const float2 x = bf16x2_to_float2(v);
  return pack_bf16x2(fmaf(x.x, co, -x.y * si), fmaf(x.x, si, x.y * co));
}

__device__ __forceinline__ uint4 rotate_chunk(uint4 raw, float4 a, float4 b) {
  return make_uint4(rot2(raw.x, a.x, a.y), rot2(raw.y, a.z, a.w),
                    rot2(raw.z, b.x, b.y), rot2(raw.w, b.z, b.w));
}

__global__ void __launch_bounds__(kThreads) rope3d_kernel(RopeArgs a) {
  const int lane = threadIdx.x & 31;
  const int c = lane & 15;        // 16-byte chunk within a head row
  const int hsub = lane >> 4;     // head parity handled by this half-warp
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * kWarps;
  const int hw = a.H * a.W;
  for (int64_t tok = static_cast<int64_t>(blockIdx.x) * kWarps +
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
    const int64_t row0 = tok * a.heads;  // first head row of this token
    // Batches of kBatch head rows per lane: all loads of a batch are issued
    // before any rotation so that 2 * kBatch 16-byte loads are in flight.
    for (int hh0 = hsub; hh0 < a.heads; hh0 += 2 * kBatch) {
      uint4 vq[kBatch], vk[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int hh = hh0 + 2 * u;
        const int64_t idx = (row0 + hh) * 16 + c;
        if (hh < a.heads) {
          if (a.q) vq[u] = a.q[idx];
          if (a.k) vk[u] = a.k[idx];
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int hh = hh0 + 2 * u;
        const int64_t idx = (row0 + hh) * 16 + c;
        if (hh < a.heads) {
          if (a.q) a.q[idx] = rotate_chunk(vq[u], cs0, cs1);
          if (a.k) a.k[idx] = rotate_chunk(vk[u], cs0, cs1);
        }
      }
    }
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
  a.L = g.F * g.H * g.W;
  a.tokens = static_cast<int64_t>(B) * a.L;
  a.heads = heads;
  a.F = g.F;
  a.H = g.H;
  a.W = g.W;
  int64_t blocks = (a.tokens + wan::kWarps - 1) / wan::kWarps;
  const int64_t cap = static_cast<int64_t>(sm_count[dev]) * 8;
  if (blocks > cap) blocks = cap;
  wan::rope3d_kernel<<<static_cast<unsigned>(blocks), wan::kThreads, 0,
                       wan::as_stream(s)>>>(a);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}
