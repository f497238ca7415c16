// wan_host.cu -- host-side calls of libwan: status strings, token-grid and
// sigma-schedule arithmetic, the RoPE cos/sin table, and the device check.
#include <math.h>

#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "wan_internal.cuh"

namespace wan {

int check_device(int* device_out) {
  static std::mutex mu;
  static int cached[64];  // 0 = unknown, 1 = ok, 2 = unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WAN_ECUDA;
  if (device_out) *device_out = dev;
  if (dev < 0 || dev >= 64) return WAN_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor,
                               dev) != cudaSuccess)
      return WAN_ECUDA;
    cached[dev] = (major == 10) ? 1 : 2;
  }
  return cached[dev] == 1 ? WAN_OK : WAN_EUNSUPPORTED;
}

int resident_grid(const void* kernel, int threads, int dev) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(kernel, dev);
  const auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads,
                                                    0) != cudaSuccess ||
      sms < 1 || per_sm < 1)
    return 0;
  const int grid = sms * (per_sm < 8 ? per_sm : 8);
  cache[key] = grid;
  return grid;
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType,
                                  cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                         cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

int make_map_bf16(CUtensorMap* m, const void* base, int B, int L, int heads,
                  int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return WAN_ECUDA;
  if (box_rows < 1 || box_rows > 256) return WAN_EINVAL;
  constexpr int HD = 128;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(HD),
                        static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(B)};
  // byte strides of dims 1..3 (heads, L, B)
  const cuuint64_t row = static_cast<cuuint64_t>(heads) * HD * 2;
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(HD) * 2, row,
                           row * static_cast<cuuint64_t>(L)};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WAN_OK : WAN_EINVAL;
}

}  // namespace wan

extern "C" {

const char* wan_status_string(int status) {
  switch (status) {
    case WAN_OK:
      return "ok";
    case WAN_EINVAL:
      return "invalid argument";
    case WAN_EALIGN:
      return "pointer not 16-byte aligned";
    case WAN_EUNSUPPORTED:
      return "device is not sm_100 (B200 class)";
    case WAN_ECUDA:
      return "CUDA runtime error";
    case WAN_ETIMEOUT:
      return "bounded in-kernel wait timed out";
    case WAN_ENOSPACE:
      return "needs more scratch than the library's fixed array holds";
    default:
      return "unknown status";
  }
}

int wan_version(void) { return 100; }

// Latent shape (16, (frames-1)/4 + 1, height/8, width/8) from the VAE
// strides (4, 8, 8); token grid after the (1, 2, 2) patchify.
int wan_token_grid(int frames, int height, int width, int32_t* latent_out,
                   wan_grid_t* grid_out) {
  if (!grid_out) return WAN_EINVAL;
  if (frames < 1 || (frames - 1) % 4 != 0) return WAN_EINVAL;
  if (height < 16 || width < 16 || height % 16 != 0 || width % 16 != 0)
    return WAN_EINVAL;
  const int lat_f = (frames - 1) / 4 + 1;
  const int lat_h = height / 8;
  const int lat_w = width / 8;
  if (latent_out) {
    latent_out[0] = 16;
    latent_out[1] = lat_f;
    latent_out[2] = lat_h;
    latent_out[3] = lat_w;
  }
  grid_out->F = lat_f;
  grid_out->H = lat_h / 2;
  grid_out->W = lat_w / 2;
  return WAN_OK;
}

int wan_fm_sigmas(int n_steps, double shift, double s_max,
                  double* sigmas_out) {
  if (!sigmas_out || n_steps < 1 || !(shift > 0.0) || !(s_max > 0.0) ||
      s_max > 1.0)
    return WAN_EINVAL;
  for (int i = 0; i < n_steps; ++i) {
    const double s = s_max * (1.0 - static_cast<double>(i) / n_steps);
    sigmas_out[i] = shift * s / (1.0 + (shift - 1.0) * s);
  }
  sigmas_out[n_steps] = 0.0;
  return WAN_OK;
}

size_t wan_rope3d_table_bytes(wan_grid_t g, int head_dim) {
  if (head_dim != 128 || g.F < 1 || g.H < 1 || g.W < 1 || g.F > 1024 ||
      g.H > 1024 || g.W > 1024)
    return 0;
  return static_cast<size_t>(g.F + g.H + g.W) * 22 * 2 * sizeof(float);
}

// Rows of 22 {cos, sin} pairs: time band (pairs j = 0..21 of a 44-channel
// band), height band (j = 0..20 of 42, pad last), width band (pad first,
// then j = 0..20).  Angles pos * theta^(-2j / D_band) are formed and turned
// into cos / sin in fp64, then rounded once to fp32.
int wan_rope3d_table(wan_grid_t g, int head_dim, double theta, void* d_table,
                     size_t bytes, void* s) {
  const size_t need = wan_rope3d_table_bytes(g, head_dim);
  if (need == 0 || !d_table || bytes < need || !(theta > 0.0))
    return WAN_EINVAL;
  if (!wan::aligned16(d_table)) return WAN_EALIGN;
  int st = wan::check_device(nullptr);
  if (st != WAN_OK) return st;
  std::vector<float> host(need / sizeof(float));
  auto put = [&](int row, int e, double angle) {
    host[(static_cast<size_t>(row) * 22 + e) * 2 + 0] =
        static_cast<float>(cos(angle));
    host[(static_cast<size_t>(row) * 22 + e) * 2 + 1] =
        static_cast<float>(sin(angle));
  };
  const int widths[3] = {head_dim - 4 * (head_dim / 6), 2 * (head_dim / 6),
                         2 * (head_dim / 6)};  // 44, 42, 42
  const int sides[3] = {g.F, g.H, g.W};
  const int first_entry[3] = {0, 0, 1};
  int row = 0;
  for (int band = 0; band < 3; ++band) {
    const int D = widths[band];
    for (int pos = 0; pos < sides[band]; ++pos, ++row) {
      for (int e = 0; e < 22; ++e) put(row, e, 0.0);  // pads: {1, 0}
      for (int j = 0; j < D / 2; ++j) {
        const double inv_freq = pow(theta, -2.0 * j / D);
        put(row, first_entry[band] + j, static_cast<double>(pos) * inv_freq);
      }
    }
  }
  // Pageable source: the copy is staged before cudaMemcpyAsync returns, so
  // the vector may be released right after.
  if (cudaMemcpyAsync(d_table, host.data(), need, cudaMemcpyHostToDevice,
                      wan::as_stream(s)) != cudaSuccess)
    return WAN_ECUDA;
  return WAN_OK;
}

}  // extern "C"
