// attention.cu -- flash-style attention forward for sm_100a (tcgen05 / TMEM /
// TMA), used for both the full spatio-temporal self-attention (optionally
// with the 3D RoPE fused into the Q / K tile stage) and the length-masked
// cross-attention to text.
//
// Wan2.2 source reading, ch. 4 "Full forward of one block" and ch. 8 "What
// is 75600^2": O = softmax(Q K^T / sqrt(d)) V over all tokens, two matrix
// products per head; ch. 3 "Where did the prompt go": text keys past each
// prompt's true length take no part.  Wan paper explainer, section "Text
// encoder": softmax(Q K_text^T / sqrt(d_k)) V_text.
//
// One CTA per (128-row query tile, head, batch row).  Warp roles:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r); reads a
//              128x128 fp32 score tile from TMEM, keeps the running row max
//              and sum, writes P (bf16) back into TMEM over the scores it
//              came from, rescales the O accumulator in TMEM when the max
//              grows by more than 2^8, and runs the epilogue (O / l -> bf16).
//   warp 4     TMA producer: Q tile once, then K / V tiles through an
//              NS-stage ring.
//   warp 5     MMA issuer (one elected lane): S = Q K^T (SS form, both
//              operands K-major in smem) into one of two TMEM score buffers,
//              O += P V (TS form, P from TMEM, V MN-major in smem).
//   warps 6-7  (RoPE variant only) rotate the Q tile and every K tile in
//              shared memory before the tensor cores read them (two rows
//              per thread; 8 warps keep the 255-register cap per thread).
// Tensor memory: columns [0,128) and [128,256) score / P buffers (double
// buffered so S(j+1) runs while row j's softmax works), [256,384) O.
// Tiles are stored as two 64-column halves, each [128 rows][128 B] with the
// 128-byte swizzle TMA writes and UMMA reads.
#include <math.h>

#include <mutex>

#include "wan_internal.cuh"

namespace wan {

__device__ int g_wan_status = 0;

namespace {

constexpr int BM = 128;                      // query rows per tile
constexpr int BN = 128;                      // keys per block
constexpr int HD = 128;                      // head dim
constexpr int NS = 3;                        // K / V ring stages
constexpr uint32_t HALF = 16384;             // one [128][64] bf16 half tile
constexpr uint32_t TILE = 2 * HALF;          // one [128][128] bf16 tile
constexpr uint32_t SMEM_DYN = TILE * (1 + 2 * NS) + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_O = 256;               // O accumulator column
constexpr int MAX_CROSS_BATCH = 512;
constexpr int kRopeThreads = 64;             // warps 6-7 of the RoPE variant
constexpr float RESCALE_LOG2 = 8.0f;         // rescale O when max grows > 2^8

constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, 0);   // K-major B
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, 1);  // MN-major B

struct AttnArgs {
  __nv_bfloat16* o;
  const float4* table;  // RoPE rows of 11 float4, or null
  int Lq, Lk, heads;
  int F, H, W;          // token grid of the RoPE variant
  float scale_log2;     // softmax_scale * log2(e)
  int cross;            // 1: per-batch key length from lens[]
  int lens[MAX_CROSS_BATCH];
};

// Barrier slots.
enum : int {
  B_QFULL = 0,
  B_QREADY = 1,
  B_KFULL = 2,
  B_KREADY = B_KFULL + NS,
  B_VFULL = B_KREADY + NS,
  B_KEMPTY = B_VFULL + NS,
  B_VEMPTY = B_KEMPTY + NS,
  B_SFULL = B_VEMPTY + NS,  // 2
  B_PFULL = B_SFULL + 2,    // 2
  B_ODONE = B_PFULL + 2,
  B_OFINAL = B_ODONE + 1,   // the last PV only (single phase)
  B_DRAIN = B_OFINAL + 1,
  NBAR = B_DRAIN + 1
};

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
  float2 r;
  r.x = __uint_as_float(v << 16);
  r.y = __uint_as_float(v & 0xFFFF0000u);
  return r;
}

// Rotate row r of a swizzled [128][128] bf16 tile in shared memory by the
// 3D RoPE of token n.  Pair p = 4c + i of logical 16-byte chunk c sits at
// physical chunk c ^ (r & 7) of the row's half.
__device__ __forceinline__ void rope_row(uint8_t* tile, int r, int n,
                                         const AttnArgs& a) {
  const int hw = a.H * a.W;
  const int f = n / hw;
  const int h = (n / a.W) % a.H;
  const int w = n % a.W;
  const float4* tt = a.table + f * 11;
  const float4* th = a.table + (a.F + h) * 11;
  const float4* tw = a.table + (a.F + a.H + w) * 11;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    uint4* p = reinterpret_cast<uint4*>(tile + (c >> 3) * HALF + r * 128 +
                                        (((c & 7) ^ (r & 7)) << 4));
    uint4 raw = *p;
    uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int p0 = 4 * c + 2 * half;
      float4 cs;
      if (p0 + 1 < 22) {
        cs = __ldg(tt + (p0 >> 1));
      } else if (p0 >= 22 && p0 + 1 < 43) {
        cs = __ldg(th + ((p0 - 22) >> 1));
      } else if (p0 >= 44) {
        cs = __ldg(tw + ((p0 - 42) >> 1));
      } else {
        const float4 lo = __ldg(th + 10);
        const float4 hi = __ldg(tw);
        cs = make_float4(lo.x, lo.y, hi.z, hi.w);
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float2 v = bf16x2_to_float2(wv[2 * half + e]);
        const float co = e ? cs.z : cs.x;
        const float si = e ? cs.w : cs.y;
        wv[2 * half + e] = pack_bf16x2(fmaf(v.x, co, -v.y * si),
                                       fmaf(v.x, si, v.y * co));
      }
    }
    *p = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }
}

template <int kRope>
__global__ void __launch_bounds__(kRope ? 256 : 192, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ AttnArgs args) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar[NBAR];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * BM;
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int kv_len = args.cross ? args.lens[b] : args.Lk;
  const int nblk = (kv_len + BN - 1) / BN;
  volatile int* abort_flag = &s_abort;
  int* status = &g_wan_status;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = sm;
  uint8_t* sK = sm + TILE;
  uint8_t* sV = sK + NS * TILE;

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(&bar[B_QFULL], 1);
    mbar_init(&bar[B_QREADY], kRopeThreads);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&bar[B_KFULL + i], 1);
      mbar_init(&bar[B_KREADY + i], kRopeThreads);
      mbar_init(&bar[B_VFULL + i], 1);
      mbar_init(&bar[B_KEMPTY + i], 1);
      mbar_init(&bar[B_VEMPTY + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[B_SFULL + i], 1);
      mbar_init(&bar[B_PFULL + i], 4);
    }
    mbar_init(&bar[B_ODONE], 1);
    mbar_init(&bar[B_OFINAL], 1);
    mbar_init(&bar[B_DRAIN], 1);
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc(&s_tmem, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 4) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
    }
    bool ok = true;
    int nk = 0, nv = 0;  // K / V tiles issued
    if (lane == 0) {
      mbar_expect_tx(&bar[B_QFULL], TILE);
      tma_load_4d(sQ, &tm_q, &bar[B_QFULL], 0, head, q0, b);
      tma_load_4d(sQ + HALF, &tm_q, &bar[B_QFULL], 64, head, q0, b);
    }
    for (int j = 0; j < nblk && ok; ++j) {
      const int st = j % NS;
      const int use = j / NS;
      if (use > 0) ok = wait_warp(&bar[B_KEMPTY + st], (use - 1) & 1,
                                  abort_flag, status);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(&bar[B_KFULL + st], TILE);
        tma_load_4d(sK + st * TILE, &tm_k, &bar[B_KFULL + st], 0, head,
                    j * BN, b);
        tma_load_4d(sK + st * TILE + HALF, &tm_k, &bar[B_KFULL + st], 64,
                    head, j * BN, b);
      }
      ++nk;
      if (use > 0) ok = wait_warp(&bar[B_VEMPTY + st], (use - 1) & 1,
                                  abort_flag, status);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(&bar[B_VFULL + st], TILE);
        tma_load_4d(sV + st * TILE, &tm_v, &bar[B_VFULL + st], 0, head,
                    j * BN, b);
        tma_load_4d(sV + st * TILE + HALF, &tm_v, &bar[B_VFULL + st], 64,
                    head, j * BN, b);
      }
      ++nv;
      __syncwarp();
    }
    if (*abort_flag) {
      // Let copies already issued land before the CTA leaves.
      wait_warp_drain(&bar[B_QFULL], 0, status);
      for (int j = (nk > NS ? nk - NS : 0); j < nk; ++j)
        wait_warp_drain(&bar[B_KFULL + j % NS], (j / NS) & 1, status);
      for (int j = (nv > NS ? nv - NS : 0); j < nv; ++j)
        wait_warp_drain(&bar[B_VFULL + j % NS], (j / NS) & 1, status);
    }
  } else if (warp == 5) {
    // -------------------------------------------------------- MMA issuer --
    const uint32_t sQa = smem_u32(sQ);
    const uint32_t sKa = smem_u32(sK);
    const uint32_t sVa = smem_u32(sV);
    bool ok = wait_warp(&bar[kRope ? B_QREADY : B_QFULL], 0, abort_flag,
                        status);
    auto issue_pv = [&](int i) -> bool {
      const int pb = i & 1;
      const int st = i % NS;
      if (!wait_warp(&bar[B_PFULL + pb], (i >> 1) & 1, abort_flag, status))
        return false;
      if (!wait_warp(&bar[B_VFULL + st], (i / NS) & 1, abort_flag, status))
        return false;
      if (args.cross && kv_len < (i + 1) * BN) {
        // Text padding rows may hold anything (NaN included): P is 0 there
        // but 0 * NaN is not, so clear those V rows before the MMA.
        const int first = kv_len - i * BN;
        uint8_t* vt = sV + st * TILE;
        for (int idx = lane; idx < (BN - first) * 16; idx += 32) {
          const int r = first + (idx >> 4);
          const int c = idx & 15;
          *reinterpret_cast<uint4*>(vt + (c >> 3) * HALF + r * 128 +
                                    ((c & 7) << 4)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          // B = V[16k .. 16k+15][0..127]: MN-major, 8-key groups 1024 B
          // apart (SBO), the two 64-column halves 16 KB apart (LBO).
          const uint64_t bdesc =
              sdesc_sw128(sVa + st * TILE + k * 2048, HALF, 1024);
          umma_ts(tmem + TM_O, tmem + pb * 128 + k * 8, bdesc, IDESC_PV,
                  (i > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&bar[B_ODONE]);
        umma_commit(&bar[B_VEMPTY + st]);
        if (i == nblk - 1) umma_commit(&bar[B_OFINAL]);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < nblk && ok; ++j) {
      const int st = j % NS;
      ok = wait_warp(&bar[(kRope ? B_KREADY : B_KFULL) + st], (j / NS) & 1,
                     abort_flag, status);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sbuf = tmem + (j & 1) * 128;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          // K-major operands: 16-element K slices are 32 B apart inside a
          // 128-B swizzle row; the second 64-column half starts 16 KB on.
          const uint32_t off = (k >> 2) * HALF + (k & 3) * 32;
          const uint64_t adesc = sdesc_sw128(sQa + off, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(sKa + st * TILE + off, 16, 1024);
          umma_ss(sbuf, adesc, bdesc, IDESC_S, k > 0 ? 1u : 0u);
        }
        umma_commit(&bar[B_SFULL + (j & 1)]);
        umma_commit(&bar[B_KEMPTY + st]);
      }
      __syncwarp();
      if (j >= 1) ok = issue_pv(j - 1);
    }
    if (ok) ok = issue_pv(nblk - 1);
    // Drain every MMA before tensor memory is released.
    if (lane == 0) umma_commit(&bar[B_DRAIN]);
    __syncwarp();
    wait_warp_drain(&bar[B_DRAIN], 0, status);
  } else if (warp < 4) {
    // ----------------------------------------------------------- softmax --
    const int r = threadIdx.x;  // query row in the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c2 = args.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int sb = j & 1;
      ok = wait_warp(&bar[B_SFULL + sb], (j >> 1) & 1, abort_flag, status);
      if (!ok) break;
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + sb * 128 + c * 32, s + c * 32);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_wait32(s + c * 32);
      const int lim = kv_len - j * BN;  // valid keys in this block
      if (lim < BN) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < BN; ++c) mx = fmaxf(mx, s[c]);
      mx *= c2;
      bool need = false;
      if (j == 0) {
        m_run = mx;
      } else {
        need = mx > m_run + RESCALE_LOG2;
      }
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m_run;
        const float alpha = ex2(m_run - m_new);
        // O holds blocks 0..j-1 only after PV(j-1) has completed.
        ok = wait_warp(&bar[B_ODONE], (j - 1) & 1, abort_flag, status);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(lane_base + TM_O + c * 32, o);
          tmem_ld_wait32(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(lane_base + TM_O + c * 32, o);
        }
        tmem_st_wait();
        l_run *= alpha;
        m_run = m_new;
      }
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(fmaf(s[c * 32 + 2 * e], c2, -m_run));
          const float p1 = ex2(fmaf(s[c * 32 + 2 * e + 1], c2, -m_run));
          sum += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        // P (bf16 pairs) over the first 64 columns of this score buffer.
        tmem_st16(lane_base + sb * 128 + c * 16, pk);
      }
      l_run += sum;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_PFULL + sb]);
    }
    // ODONE may be two phases behind here (only PV(nblk-3) is implied by
    // the last score tile), so the final PV has a barrier of its own.
    if (ok) ok = wait_warp(&bar[B_OFINAL], 0, abort_flag, status);
    if (ok) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      const int row = q0 + r;
      __nv_bfloat16* orow =
          args.o + ((static_cast<int64_t>(b) * args.Lq + row) * args.heads +
                    head) * HD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(lane_base + TM_O + c * 32, o);
        tmem_ld_wait32(o);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(o[2 * e] * inv, o[2 * e + 1] * inv);
        if (row < args.Lq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2],
                                pk[4 * e + 3]);
        }
      }
    }
  } else if (kRope) {
    // -------------------------------------------------------------- RoPE --
    const int t = threadIdx.x - 192;  // rows t and t + 64 of each tile
    bool ok = wait_warp(&bar[B_QFULL], 0, abort_flag, status);
    if (ok) {
      for (int r = t; r < BM; r += kRopeThreads)
        if (q0 + r < args.Lq) rope_row(sQ, r, q0 + r, args);
      fence_proxy_async_smem();
      mbar_arrive(&bar[B_QREADY]);
    }
    for (int j = 0; j < nblk && ok; ++j) {
      const int st = j % NS;
      ok = wait_warp(&bar[B_KFULL + st], (j / NS) & 1, abort_flag, status);
      if (!ok) break;
      for (int r = t; r < BN; r += kRopeThreads)
        if (j * BN + r < kv_len) rope_row(sK + st * TILE, r, j * BN + r, args);
      fence_proxy_async_smem();
      mbar_arrive(&bar[B_KREADY + st]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host --

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

// Tensor map of a [B, L, heads, 128] bf16 tensor with a [1][128][1][64] box
// (128 tokens x 64 channels of one head), 128-byte swizzle, zero fill past L.
int make_map(CUtensorMap* m, const void* base, int B, int L, int heads) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return WAN_ECUDA;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(HD),
                        static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(B)};
  // byte strides of dims 1..3 (heads, L, B)
  const cuuint64_t row = static_cast<cuuint64_t>(heads) * HD * 2;
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(HD) * 2, row,
                           row * static_cast<cuuint64_t>(L)};
  cuuint32_t box[4] = {64, 1, BM, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? WAN_OK : WAN_EINVAL;
}

template <int kRope>
int launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
           const AttnArgs& a, int B, cudaStream_t s) {
  static std::mutex mu;
  static bool attr_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return WAN_ECUDA;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(attn_fwd_kernel<kRope>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMEM_DYN) != cudaSuccess)
        return WAN_ECUDA;
      attr_set[dev] = true;
    }
  }
  dim3 grid((a.Lq + BM - 1) / BM, a.heads, B);
  attn_fwd_kernel<kRope><<<grid, kRope ? 256 : 192, SMEM_DYN, s>>>(mq, mk, mv,
                                                                   a);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}

int check_common(const void* q, const void* k, const void* v, void* o, int B,
                 int Lq, int Lk, int heads, int head_dim,
                 float softmax_scale) {
  if (!q || !k || !v || !o) return WAN_EINVAL;
  if (head_dim != HD || B < 1 || Lq < 1 || Lk < 1 || heads < 1)
    return WAN_EINVAL;
  if (heads > 65535 || B > 65535 || Lq > (1 << 26) || Lk > (1 << 26))
    return WAN_EINVAL;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return WAN_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return WAN_EALIGN;
  if (o == q || o == k || o == v) return WAN_EINVAL;
  return WAN_OK;
}

}  // namespace
}  // namespace wan

extern "C" {

int wan_self_attn(const void* q, const void* k, const void* v, void* o,
                  int B, wan_grid_t g, int heads, int head_dim,
                  const void* d_table, float softmax_scale, void* s) {
  using namespace wan;
  if (g.F < 1 || g.H < 1 || g.W < 1) return WAN_EINVAL;
  const int64_t L64 = static_cast<int64_t>(g.F) * g.H * g.W;
  if (L64 > (1 << 26)) return WAN_EINVAL;
  const int L = static_cast<int>(L64);
  int st = check_common(q, k, v, o, B, L, L, heads, head_dim, softmax_scale);
  if (st != WAN_OK) return st;
  if (d_table) {
    if (wan_rope3d_table_bytes(g, head_dim) == 0) return WAN_EINVAL;
    if (!aligned16(d_table)) return WAN_EALIGN;
  }
  st = check_device(nullptr);
  if (st != WAN_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, q, B, L, heads)) != WAN_OK) return st;
  if ((st = make_map(&mk, k, B, L, heads)) != WAN_OK) return st;
  if ((st = make_map(&mv, v, B, L, heads)) != WAN_OK) return st;
  AttnArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.table = static_cast<const float4*>(d_table);
  a.Lq = L;
  a.Lk = L;
  a.heads = heads;
  a.F = g.F;
  a.H = g.H;
  a.W = g.W;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.cross = 0;
  return d_table ? launch<1>(mq, mk, mv, a, B, as_stream(s))
                 : launch<0>(mq, mk, mv, a, B, as_stream(s));
}

int wan_cross_attn(const void* q, const void* k_ctx, const void* v_ctx,
                   void* o, const int32_t* ctx_lens, int B, int Lq, int Lk,
                   int heads, int head_dim, float softmax_scale, void* s) {
  using namespace wan;
  int st = check_common(q, k_ctx, v_ctx, o, B, Lq, Lk, heads, head_dim,
                        softmax_scale);
  if (st != WAN_OK) return st;
  if (!ctx_lens || B > MAX_CROSS_BATCH) return WAN_EINVAL;
  for (int i = 0; i < B; ++i)
    if (ctx_lens[i] < 1 || ctx_lens[i] > Lk) return WAN_EINVAL;
  st = check_device(nullptr);
  if (st != WAN_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, q, B, Lq, heads)) != WAN_OK) return st;
  if ((st = make_map(&mk, k_ctx, B, Lk, heads)) != WAN_OK) return st;
  if ((st = make_map(&mv, v_ctx, B, Lk, heads)) != WAN_OK) return st;
  AttnArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.table = nullptr;
  a.Lq = Lq;
  a.Lk = Lk;
  a.heads = heads;
  a.F = a.H = a.W = 1;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.cross = 1;
  for (int i = 0; i < B; ++i) a.lens[i] = ctx_lens[i];
  return launch<0>(mq, mk, mv, a, B, as_stream(s));
}

int wan_device_status(int clear) {
  int st = wan::check_device(nullptr);
  if (st != WAN_OK) return st;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, wan::g_wan_status, sizeof(int)) != cudaSuccess)
    return WAN_ECUDA;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(wan::g_wan_status, &zero, sizeof(int)) !=
        cudaSuccess)
      return WAN_ECUDA;
  }
  return v;
}

}  // extern "C"
