// transpose.cu -- block transpose of rows: out[j][i][:] = in[i][j][:], the
// layout move on either side of the Ulysses all-to-all.
//
// Wan2.2 source reading, ch. 8 "Ulysses": attention cannot cut the
// sequence, so each rank trades its sequence shard of every head for the
// whole sequence of its share of the heads with one all-to-all (scatter one
// dimension, gather another), runs attention, and trades back; heads must
// divide by the rank count.  With q/k/v/o laid out [B, L, heads, 128], a
// rank's outgoing chunks and incoming shards are contiguous only after an
// outer-dimension swap of whole rows:
//   before the exchange, [B * Ls][P][Hp * 256 B] -> [P][B * Ls][Hp * 256 B]
//   after it (B > 1),    [P][B][Ls * Hp * 256 B] -> [B][P][Ls * Hp * 256 B]
// and the mirror images on the way back.  HBM-bound: every byte is read and
// written once; 16-byte vector accesses, rows copied by consecutive threads.
#include "wan_internal.cuh"

namespace wan {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// One warp per output row (j, i): one division per row, lanes copy
// consecutive 16-byte chunks, four loads in flight per lane.
__global__ void __launch_bounds__(kThreads)
    transpose_blocks_kernel(const uint4* __restrict__ in,
                            uint4* __restrict__ out, int64_t a, int64_t b,
                            int64_t row16) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = a * b;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * kWarps +
                   (threadIdx.x >> 5);
       r < rows; r += wstride) {
    const int64_t j = r / a;
    const int64_t i = r - j * a;
    const uint4* src = in + (i * b + j) * row16;
    uint4* dst = out + r * row16;
    // up to four loads in flight per lane before the stores
    for (int64_t c0 = lane; c0 < row16; c0 += 4 * 32) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + u * 32 < row16) v[u] = src[c0 + u * 32];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + u * 32 < row16) dst[c0 + u * 32] = v[u];
    }
  }
}

}  // namespace
}  // namespace wan

extern "C" int wan_transpose_blocks(const void* in, void* out, int64_t a,
                                    int64_t b, int64_t row_bytes, void* s) {
  if (a < 0 || b < 0 || row_bytes < 0 || row_bytes % 16 != 0)
    return WAN_EINVAL;
  if (a == 0 || b == 0 || row_bytes == 0) return WAN_OK;
  if (!in || !out) return WAN_EINVAL;
  if (!wan::aligned16(in) || !wan::aligned16(out)) return WAN_EALIGN;
  // no overlap: the move is out of place
  const uintptr_t pi = reinterpret_cast<uintptr_t>(in);
  const uintptr_t po = reinterpret_cast<uintptr_t>(out);
  const uintptr_t n = static_cast<uintptr_t>(a * b * row_bytes);
  if (pi < po + n && po < pi + n) return WAN_EINVAL;
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
  const int64_t row16 = row_bytes / 16;
  int64_t blocks = (a * b + wan::kWarps - 1) / wan::kWarps;
  const int64_t cap = static_cast<int64_t>(sm_count[dev]) * 8;
  if (blocks > cap) blocks = cap;
  wan::transpose_blocks_kernel<<<static_cast<unsigned>(blocks), wan::kThreads,
                                 0, wan::as_stream(s)>>>(
      static_cast<const uint4*>(in), static_cast<uint4*>(out), a, b, row16);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}
