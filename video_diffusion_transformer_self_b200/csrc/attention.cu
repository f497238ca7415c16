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
// Work items are (256 query rows = two 128-row tiles, head, batch row); a CTA
// runs one item, or, for cross-attention, walks items persistently (one CTA
// per SM) so that the next item's Q loads while the current one drains.  The
// two tiles ping-pong: while the softmax of one tile runs, the tensor cores
// run the other tile's P V and next Q K^T, so neither waits on the other.
// Warp roles (384 threads, registers rebalanced with setmaxnreg):
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1: thread r owns query row r
//              (TMEM lane r).  Reads the 128x128 fp32 score tile from TMEM,
//              keeps the running row max (log2 units) and sum, rescales O
//              in TMEM when the max grows by more than 2^8 (exact after the
//              final O / l), writes P (bf16) back into TMEM over its
//              scores, and writes the bf16 epilogue.  A quarter of the
//              exponentials run on the FMA pipe (exp2_fma2) to offload the
//              MUFU unit.
//   warp 8     TMA producer: each item's two Q tiles, then K (3-stage ring) and
//              V (2-stage ring).
//   warp 9     MMA issuer (one lane): S_t = Q_t K^T (both operands K-major in
//              smem) and O_t += P_t V (P from TMEM, V MN-major in smem), in
//              the order PV_0(j-1), S_0(j), PV_1(j-1), S_1(j).  Measured:
//              tcgen05.mma issue slows from 64 to 89 cycles per MMA while
//              FMA work fills this warp's sub-partition (MUFU or integer
//              work there, or FMA work on another sub-partition, does not
//              slow it), so the 16 MMAs that follow each softmax sit on the
//              tile's critical path.  A second issuer warp measured slower.
//   warps 10-11  RoPE variants: rotate the Q tiles (kRope 1 and 2) and every
//              K tile (kRope 1) in shared memory before the tensor cores read
//              them; with kRope 2, K comes in rotated by the RoPE pass.
// Tensor memory (512 columns): S/P of tile 0 at 0, of tile 1 at 128, O of
// tile 0 at 256, of tile 1 at 384.  Operand tiles are [128 rows][128 ch]
// bf16 stored as two 64-channel halves of [128][128 B] with the 128-byte
// swizzle that TMA writes and UMMA reads.
#include <math.h>

#include <mutex>

#include "wan_internal.cuh"

namespace wan {

__device__ int g_wan_status = 0;

namespace {

constexpr int BM = 128;                      // query rows per tile
constexpr int QT = 2;                        // query tiles per CTA
constexpr int BN = 128;                      // keys per block
constexpr int HD = 128;                      // head dim
constexpr int NSK = 3;                       // K ring stages
constexpr int NSV = 2;                       // V ring stages
constexpr uint32_t HALF = 16384;             // one [128][64] bf16 half tile
constexpr uint32_t TILE = 2 * HALF;          // one [128][128] bf16 tile
constexpr uint32_t SMEM_DYN = TILE * (QT + NSK + NSV) + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_O = 256;               // O of tile t at TM_O + 128 t
constexpr int kThreads = 384;
constexpr int kSoftmaxRegs = 208;            // warps 0-7
constexpr int kOtherRegs = 88;               // warps 8-11
constexpr int kRopeThreads = 64;             // warps 10-11
constexpr int MAX_CROSS_BATCH = 512;
constexpr float RESCALE_LOG2 = 8.0f;         // rescale O when max grows > 2^8
// P of a tile can be published in NPART key ranges so that P V on the
// first keys overlaps the exponentials of the rest.  Measured on B200 at
// 32,760 and 75,600 tokens: 2 parts 6% and 4 parts 20% slower than 1 (each
// publication waits for the warp's TMEM stores), so P is published whole.
constexpr int NPART = 1;
constexpr int KPP = BN / 16 / NPART;         // P V K-steps per part
static_assert(BN % (32 * NPART) == 0, "parts of whole 32-key chunks");
// Pairs (2e, 2e+1) with (e & 7) < kEmuPer8 take the FMA-pipe exponential.
constexpr int kEmuPer8 = 2;
// The same for the CTA-pair kernel's softmax.
#ifndef WAN_PAIR_EMU8
#define WAN_PAIR_EMU8 2
#endif
constexpr int kPairEmu8 = WAN_PAIR_EMU8;

constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, 0);   // K-major B
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, 1);  // MN-major B

struct AttnArgs {
  __nv_bfloat16* o;
  const float4* table;  // RoPE rows of 11 float4, or null
  int Lq, Lk, heads;
  int F, H, W;          // token grid of the RoPE variant
  float scale_log2;     // softmax_scale * log2(e)
  int cross;            // 1: per-batch key length from lens[]
  int chunk;            // > 0: block-causal, chunk length in tokens
  int q_offset;         // block-causal: absolute position of query row 0
  int n_tiles_x;        // 256-row query tile pairs per (head, batch row)
  int items;            // n_tiles_x * heads * B * n_split work items
  int n_split = 1;             // key ranges per (tile pair, head, batch)
  float* part_o = nullptr;     // n_split > 1: unnormalised O per key range,
  float2* part_ml = nullptr;   //   fp32 [split][B][Lq][heads][128], and
  int64_t split_rows = 0;      //   (row max, row sum); B * Lq * heads rows
  int lens[MAX_CROSS_BATCH];
};

// One work item: a pair of 128-row query tiles of one (head, batch row),
// and with n_split > 1 one of n_split consecutive ranges of its key blocks.
// Items are numbered key range fastest, then tile, then head, then batch
// row; block-causal items run heaviest first within a head.
struct Item {
  int q0, head, b, kv_len, nblk;
  int kb0;    // first key block of the item's range
  int split;  // index of the key range
};

__device__ __forceinline__ Item item_of(const AttnArgs& a, int it) {
  Item c;
  c.split = it % a.n_split;
  it /= a.n_split;
  const int tx = it % a.n_tiles_x;
  const int rest = it / a.n_tiles_x;
  c.head = rest % a.heads;
  c.b = rest / a.heads;
  const int tile_x = a.chunk ? (a.n_tiles_x - 1 - tx) : tx;
  c.q0 = tile_x * (QT * BM);
  int kv = a.cross ? a.lens[c.b] : a.Lk;
  if (a.chunk) {
    // keys visible to the last query row of this item
    const int last = min(c.q0 + QT * BM, a.Lq) - 1 + a.q_offset;
    kv = min(a.Lk, (last / a.chunk + 1) * a.chunk);
  }
  c.kv_len = kv;
  const int nb = (kv + BN - 1) / BN;
  c.kb0 = c.split * nb / a.n_split;
  c.nblk = (c.split + 1) * nb / a.n_split - c.kb0;
  return c;
}

// Barrier slots.
enum : int {
  B_QFULL = 0,
  B_QREADY = 1,
  B_KFULL = 2,
  B_KREADY = B_KFULL + NSK,
  B_KEMPTY = B_KREADY + NSK,
  B_VFULL = B_KEMPTY + NSK,
  B_VEMPTY = B_VFULL + NSV,
  B_SFULL = B_VEMPTY + NSV,  // per tile
  B_PPART = B_SFULL + QT,    // per tile and part, one arrival per warp
  B_OFINAL = B_PPART + QT * NPART,  // per tile: an item's last PV done
  B_OFREE = B_OFINAL + QT,   // per tile: O of the item read out (4 warps)
  B_QEMPTY = B_OFREE + QT,   // an item's S MMAs done: Q buffer reusable
  B_DRAIN = B_QEMPTY + 1,
  B_OSTAGE = B_DRAIN + 1,    // per tile: output staging buffer free
  B_OWRITTEN = B_OSTAGE + QT,  // per tile: staging written (4 warps)
  NBAR = B_OWRITTEN + QT
};

// ------------------------------------------------------- small helpers --

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
  float2 r;
  r.x = __uint_as_float(v << 16);
  r.y = __uint_as_float(v & 0xFFFF0000u);
  return r;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// 2^x for two lanes on the FMA pipe.  Cody-Waite style reduction
// x = n + f, n = round-to-nearest(x) by the 1.5 * 2^23 add (n lands in the
// low mantissa bits of j), f in [-0.5, 0.5]; 2^f by a degree-3 polynomial
// fitted here (csrc/fit_exp2.py: weighted least squares on Chebyshev nodes,
// max relative error 1.2e-4 on [-126, 8]); 2^n applied by adding n << 23 to
// the bit pattern.  x is clamped to >= -126 so the exponent cannot wrap.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  const float2 j = fadd2(x, magic);
  const float2 f = fsub2(x, fsub2(j, magic));
  float2 p = ffma2(make_float2(5.459282547e-02f, 5.459282547e-02f), f,
                   make_float2(2.422178388e-01f, 2.422178388e-01f));
  p = ffma2(p, f, make_float2(6.933686137e-01f, 6.933686137e-01f));
  p = ffma2(p, f, make_float2(1.0f, 1.0f));
  return make_float2(
      __uint_as_float(__float_as_uint(p.x) + (__float_as_uint(j.x) << 23)),
      __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(j.y) << 23)));
}

__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
}
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
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

// Max of N scores with plain 2-input max and eight independent chains:
// used for blocks whose masked entries hold -inf.
template <int N>
__device__ __forceinline__ float rowmax_masked(const float* s) {
  static_assert(N % 8 == 0 && N >= 8, "N");
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = s[i];
#pragma unroll
  for (int c = 8; c < N; ++c) m[c & 7] = fmaxf(m[c & 7], s[c]);
  return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])),
               fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

// Max of N finite scores with 3-input max and four independent chains:
// s[0..3] seed the chains, s[4..N-5] go 8 per step, s[N-4..N-1] close them.
template <int N>
__device__ __forceinline__ float rowmax(const float* s) {
  static_assert(N % 8 == 0 && N >= 16, "N");
  float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
  for (int c = 4; c + 8 <= N - 4; c += 8) {
    m0 = fmax3(m0, s[c + 0], s[c + 1]);
    m1 = fmax3(m1, s[c + 2], s[c + 3]);
    m2 = fmax3(m2, s[c + 4], s[c + 5]);
    m3 = fmax3(m3, s[c + 6], s[c + 7]);
  }
  m0 = fmax3(m0, s[N - 4], s[N - 3]);
  m1 = fmax3(m1, s[N - 2], s[N - 1]);
  return fmaxf(fmax3(m0, m1, m2), m3);
}

// p = 2^(s * c2 - m) for 128 scores, packed bf16 P stored into TMEM at
// `pcol` (64 columns), sum of p returned.  kEmu: use the FMA-pipe
// exponential for part of the pairs (never for a masked block, whose -inf
// entries must give exact zeros).
template <bool kEmu, int kEmu8 = kEmuPer8>
__device__ __forceinline__ void exp_store_chunks(const float* s, float c2,
                                                 float m, uint32_t pcol,
                                                 float2 (&acc)[4], int c0,
                                                 int c1) {
  // Chunks [c0, c1) of 32 keys (constants after unrolling):
  // p = 2^(s c2 - m), packed to bf16 pairs into the tile's P columns (16 per
  // chunk), p summed into acc in fp32.
  const float2 c22 = make_float2(c2, c2);
  const float2 nm2 = make_float2(-m, -m);
#pragma unroll
  for (int c = c0; c < c1; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int pair = c * 16 + e;
      const float2 x =
          ffma2(make_float2(s[2 * pair], s[2 * pair + 1]), c22, nm2);
      float2 p;
      if (kEmu && (pair & 7) < kEmu8) {
        p = exp2_fma2(x);
      } else {
        p.x = ex2(x.x);
        p.y = ex2(x.y);
      }
      acc[e & 3] = fadd2(acc[e & 3], p);
      pk[e] = pack_bf16x2(p.x, p.y);
    }
    tmem_st16(pcol + c * 16, pk);
  }
}

// kPersist: the CTA walks items it = blockIdx.x, + gridDim.x, ...;
// otherwise it runs item blockIdx.x only (the loops below then run once and
// compile to straight-line code).
template <int kRope, int kPersist>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o,
                    const __grid_constant__ AttnArgs args) {
  // Ring depths: cross-attention (kPersist) gives one K stage to a staging
  // buffer for the output tile, which it writes with TMA stores.
  constexpr int nsk = kPersist ? NSK - 1 : NSK;
  constexpr int nsv = NSV;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar[NBAR];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Every role walks the same items, it = blockIdx.x, + gridDim.x, ...; the
  // barrier phases of the K / V rings and of S / P run on across items
  // (g counts key blocks over all of this CTA's items, n counts items).
  volatile int* abort_flag = &s_abort;
  int* status = &g_wan_status;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = sm;                   // QT tiles
  uint8_t* sK = sm + QT * TILE;       // nsk tiles
  uint8_t* sV = sK + nsk * TILE;      // nsv tiles
  uint8_t* sO = sV + nsv * TILE;      // kPersist: one [128][64] half per tile

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(&bar[B_QFULL], 1);
    mbar_init(&bar[B_QREADY], kRopeThreads);
    for (int i = 0; i < nsk; ++i) {
      mbar_init(&bar[B_KFULL + i], 1);
      mbar_init(&bar[B_KREADY + i], kRopeThreads);
      mbar_init(&bar[B_KEMPTY + i], 1);
    }
    for (int i = 0; i < nsv; ++i) {
      mbar_init(&bar[B_VFULL + i], 1);
      mbar_init(&bar[B_VEMPTY + i], 1);
    }
    for (int t = 0; t < QT; ++t) {
      mbar_init(&bar[B_SFULL + t], 1);
      for (int q = 0; q < NPART; ++q)
        mbar_init(&bar[B_PPART + t * NPART + q], 4);
      mbar_init(&bar[B_OFINAL + t], 1);
      mbar_init(&bar[B_OFREE + t], 4);
      mbar_init(&bar[B_OSTAGE + t], 1);
      mbar_init(&bar[B_OWRITTEN + t], 4);
    }
    mbar_init(&bar[B_QEMPTY], 1);
    mbar_init(&bar[B_DRAIN], 1);
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(&s_tmem, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp >= 8) {
    // Warpgroup 2: producer, MMA issuer, RoPE.  Registers handed to the
    // softmax warpgroups first (setmaxnreg must open the warpgroup's branch).
    setmaxnreg_dec();
    if (warp == 8) {
      // ------------------------------------------------------ TMA producer --
      const bool leader = elect_one();
      if (leader) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
      }
      bool ok = true;
      int nq = 0, nk = 0, nv = 0;  // Q pairs / K / V tiles issued
      for (int it = blockIdx.x, n = 0;
           it < (kPersist ? args.items : blockIdx.x + 1) && ok;
           it += gridDim.x, ++n) {
        const Item c = item_of(args, it);
        // the previous item's S MMAs must be done with the Q buffer
        if (n > 0)
          ok = wait_warp(&bar[B_QEMPTY], (n - 1) & 1, abort_flag, status);
        if (!ok) break;
        if (leader) {
          mbar_expect_tx(&bar[B_QFULL], QT * TILE);
          for (int t = 0; t < QT; ++t) {
            tma_load_4d(sQ + t * TILE, &tm_q, &bar[B_QFULL], 0, c.head,
                        c.q0 + t * BM, c.b);
            tma_load_4d(sQ + t * TILE + HALF, &tm_q, &bar[B_QFULL], 64,
                        c.head, c.q0 + t * BM, c.b);
          }
        }
        ++nq;
        for (int j = 0; j < c.nblk && ok; ++j) {
          const int g = nk;  // key blocks issued so far == this block's g
          const int sk = g % nsk, uk = g / nsk;
          if (uk > 0)
            ok = wait_warp(&bar[B_KEMPTY + sk], (uk - 1) & 1, abort_flag,
                           status);
          if (!ok) break;
          if (leader) {
            mbar_expect_tx(&bar[B_KFULL + sk], TILE);
            tma_load_4d(sK + sk * TILE, &tm_k, &bar[B_KFULL + sk], 0, c.head,
                        (c.kb0 + j) * BN, c.b);
            tma_load_4d(sK + sk * TILE + HALF, &tm_k, &bar[B_KFULL + sk], 64,
                        c.head, (c.kb0 + j) * BN, c.b);
          }
          ++nk;
          const int sv = g % nsv, uv = g / nsv;
          if (uv > 0)
            ok = wait_warp(&bar[B_VEMPTY + sv], (uv - 1) & 1, abort_flag,
                           status);
          if (!ok) break;
          if (leader) {
            mbar_expect_tx(&bar[B_VFULL + sv], TILE);
            tma_load_4d(sV + sv * TILE, &tm_v, &bar[B_VFULL + sv], 0, c.head,
                        (c.kb0 + j) * BN, c.b);
            tma_load_4d(sV + sv * TILE + HALF, &tm_v, &bar[B_VFULL + sv], 64,
                        c.head, (c.kb0 + j) * BN, c.b);
          }
          ++nv;
          __syncwarp();
        }
      }
      if (*abort_flag) {
        // Let copies already issued land before the CTA leaves.
        if (nq > 0) wait_warp_drain(&bar[B_QFULL], (nq - 1) & 1, status);
        for (int g = (nk > nsk ? nk - nsk : 0); g < nk; ++g)
          wait_warp_drain(&bar[B_KFULL + g % nsk], (g / nsk) & 1, status);
        for (int g = (nv > nsv ? nv - nsv : 0); g < nv; ++g)
          wait_warp_drain(&bar[B_VFULL + g % nsv], (g / nsv) & 1, status);
      }
    } else if (warp == 9) {
      // -------------------------------------------------------- MMA issuer --
      // Base descriptors, built once.  Per K step only a compile-time offset
      // (bytes >> 4) is added to the start-address field, which cannot carry
      // out of its 14 bits because shared addresses stay below 256 KB; this
      // keeps the single issuing thread far ahead of the tensor core.
      const uint64_t dq = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv = sdesc_sw128(smem_u32(sV), HALF, 1024);
      const bool leader = elect_one();
      // S_t(j) = Q_t K(j)^T into the score buffer of tile t.  Descriptor
      // arithmetic runs in all lanes (warp-uniform); one lane issues.
      auto issue_s = [&](int t, int g) {
        const uint64_t a0 = dq + ((t * TILE) >> 4);
        const uint64_t b0 = dk + (((g % nsk) * TILE) >> 4);
        const uint32_t d = tmem + t * 128;
        if (leader) {
#pragma unroll
          for (int k = 0; k < HD / 16; ++k) {
            // K-major operands: 16-channel K slices are 32 B apart inside a
            // 128-B swizzle row; the second 64-channel half starts 16 KB on.
            const uint32_t off = ((k >> 2) * HALF + (k & 3) * 32) >> 4;
            umma_ss(d, a0 + off, b0 + off, IDESC_S, k > 0 ? 1u : 0u);
          }
          umma_commit(&bar[B_SFULL + t]);
        }
        __syncwarp();
      };
      // O_t += P_t V over the keys of P part `part`; g is the block's global
      // count (ring stage), jl its index within the item (accumulate flag).
      auto issue_pv_part = [&](int t, int g, int jl, int part) {
        const uint64_t b0 = dv + (((g % nsv) * TILE) >> 4);
        const uint32_t d = tmem + TM_O + t * 128;
        const uint32_t a = tmem + t * 128;
        if (leader) {
          // B = V[16k .. 16k+15][0..127]: MN-major, 8-key groups 1024 B
          // apart (SBO), the two 64-channel halves 16 KB apart (LBO).
#pragma unroll
          for (int kk = 0; kk < KPP; ++kk) {
            const int k = part * KPP + kk;
            umma_ts(d, a + k * 8, b0 + ((k * 2048) >> 4), IDESC_PV,
                    (jl > 0 || k > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      // Arrive on `b` when all MMAs issued so far are done (one lane).
      auto commit = [&](uint64_t* b) {
        if (leader) umma_commit(b);
        __syncwarp();
      };
      // Waits for V of block g and clears its text-padding rows: they may
      // hold anything (NaN included), and P is 0 there but 0 * NaN is not.
      auto ready_v = [&](int g, int jl, int kv_len) -> bool {
        if (!wait_warp(&bar[B_VFULL + g % nsv], (g / nsv) & 1, abort_flag,
                       status))
          return false;
        if (args.cross && kv_len < (jl + 1) * BN) {
          const int first = kv_len - jl * BN;
          uint8_t* vt = sV + (g % nsv) * TILE;
          for (int idx = lane; idx < (BN - first) * 16; idx += 32) {
            const int r = first + (idx >> 4);
            const int c = idx & 15;
            *reinterpret_cast<uint4*>(vt + (c >> 3) * HALF + r * 128 +
                                      ((c & 7) << 4)) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        return true;
      };
      // O_t += P_t V for block g (index jl in item n), each part issued as
      // soon as the softmax warps have published it.  An item's first P V
      // overwrites O_t, so it also waits until the previous item's O_t has
      // been read out.
      auto pv = [&](int t, int g, int jl, int n) -> bool {
        if (jl == 0 && n > 0 &&
            !wait_warp(&bar[B_OFREE + t], (n - 1) & 1, abort_flag, status))
          return false;
        for (int part = 0; part < NPART; ++part) {
          if (!wait_warp(&bar[B_PPART + t * NPART + part], g & 1, abort_flag,
                         status))
            return false;
          tc_fence_after();
          issue_pv_part(t, g, jl, part);
        }
        return true;
      };
      bool ok = true;
      int g0 = 0;  // key blocks of earlier items
      for (int it = blockIdx.x, n = 0;
           it < (kPersist ? args.items : blockIdx.x + 1) && ok;
           it += gridDim.x, ++n) {
        const Item c = item_of(args, it);
        ok = wait_warp(&bar[kRope ? B_QREADY : B_QFULL], n & 1, abort_flag,
                       status);
        for (int j = 0; j < c.nblk && ok; ++j) {
          const int g = g0 + j;
          const int sk = g % nsk;
          if (j > 0) {
            ok = ready_v(g - 1, j - 1, c.kv_len) && pv(0, g - 1, j - 1, n);
            if (!ok) break;
          }
          ok = wait_warp(&bar[(kRope == 1 ? B_KREADY : B_KFULL) + sk],
                         (g / nsk) & 1, abort_flag, status);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, g);
          if (j > 0) {
            ok = pv(1, g - 1, j - 1, n);
            if (!ok) break;
            commit(&bar[B_VEMPTY + (g - 1) % nsv]);
          }
          issue_s(1, g);
          // the item's last S: the Q buffer is free once these are done
          if (j == c.nblk - 1) commit(&bar[B_QEMPTY]);
          commit(&bar[B_KEMPTY + sk]);
        }
        if (ok) {
          const int jl = c.nblk - 1, g = g0 + jl;
          ok = ready_v(g, jl, c.kv_len) && pv(0, g, jl, n);
          if (ok) {
            commit(&bar[B_OFINAL + 0]);
            ok = pv(1, g, jl, n);
          }
          if (ok) {
            commit(&bar[B_OFINAL + 1]);
            commit(&bar[B_VEMPTY + g % nsv]);
          }
        }
        g0 += c.nblk;
      }
      // Drain every MMA before tensor memory is released.
      commit(&bar[B_DRAIN]);
      wait_warp_drain(&bar[B_DRAIN], 0, status);
    } else if (kRope) {
      // -------------------------------------------------------------- RoPE --
      const int tr = threadIdx.x - 320;  // 0..63
      bool ok = true;
      int g0 = 0;
      for (int it = blockIdx.x, n = 0;
           it < (kPersist ? args.items : blockIdx.x + 1) && ok;
           it += gridDim.x, ++n) {
        const Item c = item_of(args, it);
        ok = wait_warp(&bar[B_QFULL], n & 1, abort_flag, status);
        if (!ok) break;
        for (int rr = tr; rr < QT * BM; rr += kRopeThreads) {
          const int tok = c.q0 + rr;
          if (tok < args.Lq)
            rope_row(sQ + (rr >> 7) * TILE, rr & 127, tok, args);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bar[B_QREADY]);
        // kRope == 2: K comes in already rotated; only Q is rotated here
        for (int j = 0; j < (kRope == 1 ? c.nblk : 0) && ok; ++j) {
          const int g = g0 + j, sk = g % nsk;
          ok = wait_warp(&bar[B_KFULL + sk], (g / nsk) & 1, abort_flag,
                         status);
          if (!ok) break;
          for (int rr = tr; rr < BN; rr += kRopeThreads)
            if (j * BN + rr < c.kv_len)
              rope_row(sK + sk * TILE, rr, j * BN + rr, args);
          fence_proxy_async_smem();
          mbar_arrive(&bar[B_KREADY + sk]);
        }
        g0 += c.nblk;
      }
    }
  } else {
    // ----------------------------------------------------------- softmax --
    setmaxnreg_inc();
    const int t = warp >> 2;                 // query tile of this warpgroup
    const int r = threadIdx.x & 127;         // row in the tile == TMEM lane
    const uint32_t lane_base =
        tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_col = lane_base + t * 128;
    const uint32_t o_col = lane_base + TM_O + t * 128;
    const float c2 = args.scale_log2;
    bool ok = true;
    int g0 = 0;
    for (int it = blockIdx.x, n = 0;
         it < (kPersist ? args.items : blockIdx.x + 1) && ok;
         it += gridDim.x, ++n) {
      const Item cur = item_of(args, it);
      // Keys this row may see: all kv_len, or its block-causal limit.
      int row_lim = cur.kv_len;
      if (args.chunk && cur.q0 + t * BM + r < args.Lq) {
        const int a = cur.q0 + t * BM + r + args.q_offset;
        row_lim = min(args.Lk, (a / args.chunk + 1) * args.chunk);
      }
      float m_run = -INFINITY;
      float l_run = 0.f;
      for (int j = 0; j < cur.nblk; ++j) {
        ok = wait_warp(&bar[B_SFULL + t], (g0 + j) & 1, abort_flag, status);
        if (!ok) break;
        tc_fence_after();
        float s[BN];
        static_assert(BN == 128, "one 128-column TMEM load per score row");
        tmem_ld128(s_col, s);
        tmem_ld_wait128(s);
        const int lim = row_lim - (cur.kb0 + j) * BN;  // valid keys here
        // warp-uniform: any masked row sends the warp down the exact path
        const bool masked = __any_sync(0xffffffffu, lim < BN);
        if (masked) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        const float mx = (masked ? rowmax_masked<BN>(s) : rowmax<BN>(s)) * c2;
        if (j == 0) {
          m_run = mx;
        } else {
          // Keep the running max unless some row's max grew by more than 2^8:
          // exponents then stay <= 8 (p <= 256, exact after the final O / l).
          // Otherwise rescale O in TMEM first.  S_t(j) complete implies
          // PV_t(j-1) complete (issued before it), so O holds exactly blocks
          // 0..j-1 here; the first part's arrival orders these stores before
          // PV_t(j).
          const bool need = mx > m_run + RESCALE_LOG2;
          if (__any_sync(0xffffffffu, need)) {
            const float m_new = need ? mx : m_run;
            const float alpha = ex2(m_run - m_new);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float o[32];
              tmem_ld32(o_col + c * 32, o);
              tmem_ld_wait32(o);
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float2 v =
                    ffma2(make_float2(o[e], o[e + 1]),
                          make_float2(alpha, alpha), make_float2(0.f, 0.f));
                o[e] = v.x;
                o[e + 1] = v.y;
              }
              tmem_st32(o_col + c * 32, o);
            }
            l_run *= alpha;
            m_run = m_new;
          }
        }
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // Publish P part by part: the MMA issuer starts P V on the first keys
        // while the rest are exponentiated.
        auto publish = [&](int part) {
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_PPART + t * NPART + part]);
        };
        constexpr int CPP = BN / 32 / NPART;  // 32-key chunks per part
#pragma unroll
        for (int part = 0; part < NPART; ++part) {
          // A row with no visible key yet (possible in a later key range
          // of a block-causal item) keeps m = -inf: its scores are all -inf
          // and exponentiate against 0 to exact zeros.
          if (masked)
            exp_store_chunks<false>(s, c2, m_run == -INFINITY ? 0.f : m_run,
                                    s_col, acc, part * CPP, (part + 1) * CPP);
          else
            exp_store_chunks<true>(s, c2, m_run, s_col, acc, part * CPP,
                                   (part + 1) * CPP);
          publish(part);
        }
        const float2 tsum = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
        l_run += tsum.x + tsum.y;
      }
      g0 += cur.nblk;
      if (ok) ok = wait_warp(&bar[B_OFINAL + t], n & 1, abort_flag, status);
      if (ok) {
        tc_fence_after();
        // Recompute the item's coordinates here instead of holding them in
        // registers through the key-block loop.
        int it_e = it;
        asm volatile("" : "+r"(it_e));
        const Item ce = item_of(args, it_e);
        const float inv = 1.0f / l_run;
        const int row = ce.q0 + t * BM + r;
        const int64_t orow_i =
            (static_cast<int64_t>(ce.b) * args.Lq + row) * args.heads + ce.head;
        if (kPersist) {
          // Output tile through shared memory and TMA stores, one 64-channel
          // half at a time: each thread writes its row's 128 B into the
          // tile's staging half (128-byte swizzle, the layout the tensor map
          // stores from), and warp 4t's lane 0 issues the store.  A row per
          // thread stored straight to global memory scatters every store
          // instruction over 32 rows 10 KB apart and stalls the warps on
          // the store queue; the next item's softmax then starts late.
          uint8_t* stg = sO + t * HALF;
          const bool issuer_warp = (warp & 3) == 0;
#pragma unroll 1
          for (int hc = 0; hc < 2; ++hc) {
            const int use = 2 * n + hc;
            if (issuer_warp) {
              // the previous store from this buffer has read it
              if (lane == 0) {
                if (use > 0) bulk_wait_group_read0();
                mbar_arrive(&bar[B_OSTAGE + t]);
              }
              __syncwarp();
            }
            const bool free_ok =
                wait_warp(&bar[B_OSTAGE + t], use & 1, abort_flag, status);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              float o[32];
              tmem_ld32(o_col + hc * 64 + c * 32, o);
              tmem_ld_wait32(o);
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 16; ++e)
                pk[e] = pack_bf16x2(o[2 * e] * inv, o[2 * e + 1] * inv);
              if (free_ok) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int cc = c * 4 + e;  // 16-byte chunk of the row
                  *reinterpret_cast<uint4*>(stg + r * 128 +
                                            ((cc ^ (r & 7)) << 4)) =
                      make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2],
                                 pk[4 * e + 3]);
                }
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[B_OWRITTEN + t]);
            if (issuer_warp) {
              const bool written =
                  wait_warp(&bar[B_OWRITTEN + t], use & 1, abort_flag, status);
              if (written && lane == 0) {
                tma_store_4d(&tm_o, stg, hc * 64, ce.head, ce.q0 + t * BM,
                             ce.b);
                bulk_commit_group();
              }
              __syncwarp();
            }
          }
        }
        if (!kPersist && args.n_split > 1) {
          // one key range of the row: unnormalised O and (row max, row sum)
          // for the combining pass
          const int64_t prow = ce.split * args.split_rows + orow_i;
          float4* dst = reinterpret_cast<float4*>(args.part_o + prow * HD);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(o_col + c * 32, o);
            tmem_ld_wait32(o);
            if (row < args.Lq) {
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[c * 8 + e] = make_float4(o[4 * e], o[4 * e + 1],
                                             o[4 * e + 2], o[4 * e + 3]);
            }
          }
          if (row < args.Lq) args.part_ml[prow] = make_float2(m_run, l_run);
        }
        if (!kPersist && args.n_split == 1) {
          // One item per CTA: once the item's last P V is done (OFINAL_t),
          // no MMA reads the K ring and no load fills it, so tile t's output
          // is staged in K stage t (two 64-channel halves, 128-byte swizzle)
          // and written by two TMA stores from warp 4t's lane 0.
          uint8_t* stg = sK + t * TILE;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(o_col + c * 32, o);
            tmem_ld_wait32(o);
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(o[2 * e] * inv, o[2 * e + 1] * inv);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int cc = c * 4 + e;  // 16-byte chunk of the 256-byte row
              *reinterpret_cast<uint4*>(stg + (cc >> 3) * HALF + r * 128 +
                                        (((cc & 7) ^ (r & 7)) << 4)) =
                  make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2],
                             pk[4 * e + 3]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_OWRITTEN + t]);
          if ((warp & 3) == 0) {
            const bool written =
                wait_warp(&bar[B_OWRITTEN + t], 0, abort_flag, status);
            if (written && lane == 0) {
              tma_store_4d(&tm_o, stg, 0, ce.head, ce.q0 + t * BM, ce.b);
              tma_store_4d(&tm_o, stg + HALF, 64, ce.head, ce.q0 + t * BM,
                           ce.b);
              bulk_commit_group();
            }
            __syncwarp();
          }
        }
        // O_t has been read: the next item's first P V may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_OFREE + t]);
      }
    }
  }

  // the output stores of the staging buffers are complete before the CTA
  // (and its shared memory) goes away
  if (warp < 8 && (warp & 3) == 0 && lane == 0) bulk_wait_group0();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ============================================================ CTA pairs ==
//
// Self-attention over pairs of CTAs on two SMs.  One tcgen05 MMA with
// cta_group::2 multiplies a 256-row query tile (128 rows in each CTA's
// tensor memory) by a 128-key block whose K rows (for Q K^T) and V channels
// (for P V) are split between the two CTAs' shared memory, so each SM
// stages half of every K / V block and the B operand costs each SM half the
// shared-memory bandwidth.  That frees tensor memory for a ring of three
// score slots per CTA: S(j+1) and S(j+2) are computed while the softmax of
// block j runs, and the softmax of one block never waits on the P V and
// Q K^T of the previous one (the two-tile kernel above has that chain).
//
// Per CTA (384 threads, registers rebalanced with setmaxnreg):
//   warps 0-7  softmax, two warps per TMEM lane quadrant: warp w owns query
//              rows 32 (w & 3) .. + 31 and every other key block (blocks j
//              with j % 2 == w >> 2), all 128 keys of each.  The running row
//              max passes from block to block through shared memory (an
//              mbarrier per quadrant): the warp of block j posts it right
//              after its block max, so the warp of block j+1 waits only for
//              that, not for block j's exponentials, and the two warps of a
//              sub-partition work on different blocks at once.  The warp
//              whose block raises the max by more than 2^8 rescales O (after
//              P V of the previous block); each warp keeps its own row sum
//              relative to the max it last used.
//   warp 8     TMA producer: this CTA's Q rows, its 64 keys of each K block
//              (3 blocks ahead of V) and its 64 channels of each V block.
//   warp 9     in CTA 0: the MMA issuer for the pair; in CTA 1: forwards the
//              completion of CTA 1's loads to CTA 0 (remote mbarrier arrive).
//   warps 10-11  (kRopeQ) rotate this CTA's 128 query rows by the 3D RoPE
//              once, in shared memory, before any MMA reads them; K comes
//              in already rotated.
// Tensor memory (512 columns, both CTAs): O at 0, score slot b at 128 + 128 b;
// P (bf16) of a block over the first 64 columns of its slot.
namespace pair {
constexpr int RM = 128;                    // query rows per CTA
constexpr int NSLOT = 3;                   // score / P slots
constexpr int KSTAGES = 5;                     // K stages (64 keys each)
constexpr int VSTAGES = 4;                     // V stages (64 channels each)
constexpr uint32_t QHALF = 16384;          // [128 rows][64 ch] bf16
constexpr uint32_t QTILE = 2 * QHALF;
constexpr uint32_t KHALF = 8192;           // [64 keys][64 ch] bf16
constexpr uint32_t KTILE = 2 * KHALF;
constexpr uint32_t VTILE = 16384;          // [128 keys][64 ch] bf16
constexpr uint32_t SMEM = QTILE + KSTAGES * KTILE + VSTAGES * VTILE + 1024;
constexpr int THREADS = 384;
constexpr uint32_t TM_SLOT0 = 128;
constexpr uint16_t BOTH = 3;               // multicast mask: CTAs 0 and 1
constexpr uint32_t IDESC_S2 = idesc_bf16_f32(2 * RM, BN, 0);
constexpr uint32_t IDESC_PV2 = idesc_bf16_f32(2 * RM, HD, 1);

enum : int {
  QFULL = 0,                  // this CTA's Q landed (local)
  QPEER = 1,                  // CTA 1's Q landed (CTA 0 only)
  KFULL = 2,                  // per K stage, local
  KPEER = KFULL + KSTAGES,        // per K stage, CTA 1's half landed (CTA 0)
  VFULL = KPEER + KSTAGES,
  VPEER = VFULL + VSTAGES,
  KEMPTY = VPEER + VSTAGES,       // per stage: the pair's MMAs are done with it
  VEMPTY = KEMPTY + KSTAGES,
  SFULL = VEMPTY + VSTAGES,       // per slot: S written (both CTAs)
  PREADY = SFULL + NSLOT,     // per slot: P written by the block's 8 warps
  PVDONE = PREADY + NSLOT,    // per slot: P V done (both CTAs)
  OFINAL = PVDONE + NSLOT,    // the item's last P V done (both CTAs)
  DRAIN = OFINAL + 1,         // every MMA done (both CTAs)
  XCH = DRAIN + 1,            // per lane quadrant: both row sums posted
  MCHAIN = XCH + 4,           // per lane quadrant: a block's row max posted
  QREADY = MCHAIN + 4,        // (kRopeQ) this CTA's Q rows rotated
  NUM_BARS = QREADY + 1
};
}  // namespace pair

template <int kRopeQ>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair::THREADS, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ AttnArgs args) {
  using namespace pair;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar[NUM_BARS];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ float s_xch[2][RM];     // [warp set][row]: final row sums
  __shared__ float s_mx[2][RM];      // [block parity][row]: running max

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;
  volatile int* abort_flag = &s_abort;
  int* status = &g_wan_status;

  // Same offsets in both CTAs: the MMAs address both with one descriptor.
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = sm;
  uint8_t* sK = sm + QTILE;
  uint8_t* sV = sK + KSTAGES * KTILE;

  // Work item of the pair: 256 query rows of one (head, batch row) and, with
  // n_split > 1, one of n_split consecutive ranges of their key blocks
  // (numbered key range fastest); the block-causal mode runs the tiles of a
  // head heaviest first.
  const int split = static_cast<int>(blockIdx.x >> 1) % args.n_split;
  const int item = static_cast<int>(blockIdx.x >> 1) / args.n_split;
  const int tx = item % args.n_tiles_x;
  const int head = (item / args.n_tiles_x) % args.heads;
  const int bb = item / args.n_tiles_x / args.heads;
  const int tile = args.chunk ? args.n_tiles_x - 1 - tx : tx;
  const int q0 = tile * (2 * RM) + static_cast<int>(rank) * RM;
  int kv_len = args.Lk;
  if (args.chunk) {
    // keys visible to the pair's last query row (both CTAs agree)
    const int last = min(tile * (2 * RM) + 2 * RM, args.Lq) - 1 + args.q_offset;
    kv_len = min(args.Lk, (last / args.chunk + 1) * args.chunk);
  }
  // this range's key blocks: kb0 .. kb0 + nblk - 1 (j below counts from 0)
  const int nb_all = (kv_len + BN - 1) / BN;
  const int kb0 = split * nb_all / args.n_split;
  const int nblk = (split + 1) * nb_all / args.n_split - kb0;

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(&bar[QFULL], 1);
    mbar_init(&bar[QPEER], 1);
    for (int i = 0; i < KSTAGES; ++i) {
      mbar_init(&bar[KFULL + i], 1);
      mbar_init(&bar[KPEER + i], 1);
      mbar_init(&bar[KEMPTY + i], 1);
    }
    for (int i = 0; i < VSTAGES; ++i) {
      mbar_init(&bar[VFULL + i], 1);
      mbar_init(&bar[VPEER + i], 1);
      mbar_init(&bar[VEMPTY + i], 1);
    }
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(&bar[SFULL + i], 1);
      mbar_init(&bar[PREADY + i], 8);
      mbar_init(&bar[PVDONE + i], 1);
    }
    mbar_init(&bar[OFINAL], 1);
    mbar_init(&bar[DRAIN], 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bar[XCH + i], 2);
      mbar_init(&bar[MCHAIN + i], 1);
    }
    mbar_init(&bar[QREADY], 64);
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc_pair(&s_tmem, 512);
  tc_fence_before();
  __syncthreads();
  // the peer's barriers are initialised before any remote arrive or commit
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp >= 8) setmaxnreg_dec();
  if (warp == 8) {
    // --------------------------------------------------------- producer --
    const bool el = elect_one();
    if (el) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_expect_tx(&bar[QFULL], QTILE);
      tma_load_4d(sQ, &tm_q, &bar[QFULL], 0, head, q0, bb);
      tma_load_4d(sQ + QHALF, &tm_q, &bar[QFULL], 64, head, q0, bb);
    }
    __syncwarp();
    bool ok = true;
    int nk = 0, nv = 0;
    // K of block j goes out with V of block j - NSLOT: the order the MMA
    // warp consumes them (S runs NSLOT blocks ahead of P V).
    for (int j = 0; j < nblk + NSLOT && ok; ++j) {
      if (j < nblk) {
        const int sk = j % KSTAGES;
        if (j >= KSTAGES)
          ok = wait_warp(&bar[KEMPTY + sk], ((j / KSTAGES) - 1) & 1,
                         abort_flag, status);
        if (!ok) break;
        if (el) {
          const int key0 = (kb0 + j) * BN + static_cast<int>(rank) * 64;
          mbar_expect_tx(&bar[KFULL + sk], KTILE);
          tma_load_4d(sK + sk * KTILE, &tm_k, &bar[KFULL + sk], 0, head, key0,
                      bb);
          tma_load_4d(sK + sk * KTILE + KHALF, &tm_k, &bar[KFULL + sk], 64,
                      head, key0, bb);
        }
        __syncwarp();
        ++nk;
      }
      const int jv = j - NSLOT;
      if (jv >= 0) {
        const int sv = jv % VSTAGES;
        if (jv >= VSTAGES)
          ok = wait_warp(&bar[VEMPTY + sv], ((jv / VSTAGES) - 1) & 1,
                         abort_flag, status);
        if (!ok) break;
        if (el) {
          mbar_expect_tx(&bar[VFULL + sv], VTILE);
          tma_load_4d(sV + sv * VTILE, &tm_v, &bar[VFULL + sv],
                      static_cast<int>(rank) * 64, head, (kb0 + jv) * BN,
                      bb);
        }
        __syncwarp();
        ++nv;
      }
    }
    if (*abort_flag) {
      // copies already issued land in this CTA before it leaves
      wait_warp_drain(&bar[QFULL], 0, status);
      for (int g = (nk > KSTAGES ? nk - KSTAGES : 0); g < nk; ++g)
        wait_warp_drain(&bar[KFULL + g % KSTAGES], (g / KSTAGES) & 1, status);
      for (int g = (nv > VSTAGES ? nv - VSTAGES : 0); g < nv; ++g)
        wait_warp_drain(&bar[VFULL + g % VSTAGES], (g / VSTAGES) & 1, status);
    }
  } else if (warp == 9 && !lead) {
    // ----------------------------------- CTA 1: forward load completions --
    auto fwd = [&](int full, int peer, uint32_t parity) -> bool {
      if (!wait_warp(&bar[full], parity, abort_flag, status)) return false;
      if (lane == 0)
        mbar_arrive_remote_relaxed(mapa_shared(smem_u32(&bar[peer]), 0));
      __syncwarp();
      return true;
    };
    bool ok = fwd(kRopeQ ? QREADY : QFULL, QPEER, 0);
    for (int j = 0; j < nblk + NSLOT && ok; ++j) {
      if (j < nblk)
        ok = fwd(KFULL + j % KSTAGES, KPEER + j % KSTAGES, (j / KSTAGES) & 1);
      const int jv = j - NSLOT;
      if (ok && jv >= 0)
        ok = fwd(VFULL + jv % VSTAGES, VPEER + jv % VSTAGES, (jv / VSTAGES) & 1);
    }
    // every MMA of the pair is done before this CTA's memory is released
    wait_warp_drain(&bar[DRAIN], 0, status);
  } else if (warp == 9) {
    // ---------------------------------------------- CTA 0: MMA issuer --
    const uint64_t dq = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dk = sdesc_sw128(smem_u32(sK), 16, 1024);
    // V: MN-major, one 64-channel swizzle atom per CTA, 8-key groups 1 KB
    const uint64_t dv = sdesc_sw128(smem_u32(sV), 16, 1024);
    const bool el = elect_one();
    bool ok =
        wait_warp(&bar[kRopeQ ? QREADY : QFULL], 0, abort_flag, status) &&
        wait_warp_cl(&bar[QPEER], 0, abort_flag, status);
    // S(j) = Q K(j)^T into slot j % NSLOT of both CTAs.
    auto issue_s = [&](int j) -> bool {
      const int sk = j % KSTAGES;
      const uint32_t ph = (j / KSTAGES) & 1;
      if (!wait_warp(&bar[KFULL + sk], ph, abort_flag, status) ||
          !wait_warp_cl(&bar[KPEER + sk], ph, abort_flag, status))
        return false;
      tc_fence_after();
      const uint64_t b0 = dk + ((sk * KTILE) >> 4);
      const uint32_t d = tmem + TM_SLOT0 + (j % NSLOT) * 128;
      if (el) {
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t oa = ((k >> 2) * QHALF + (k & 3) * 32) >> 4;
          const uint32_t ob = ((k >> 2) * KHALF + (k & 3) * 32) >> 4;
          umma_ss_pair(d, dq + oa, b0 + ob, IDESC_S2, k > 0 ? 1u : 0u);
        }
        umma_commit_pair(&bar[SFULL + j % NSLOT], BOTH);
        umma_commit_pair(&bar[KEMPTY + sk], BOTH);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < NSLOT && j < nblk && ok; ++j) ok = issue_s(j);
    for (int j = 0; j < nblk && ok; ++j) {
      const int sl = j % NSLOT, sv = j % VSTAGES;
      const uint32_t pv = (j / VSTAGES) & 1;
      ok = wait_warp_cl(&bar[PREADY + sl], (j / NSLOT) & 1, abort_flag,
                        status) &&
           wait_warp(&bar[VFULL + sv], pv, abort_flag, status) &&
           wait_warp_cl(&bar[VPEER + sv], pv, abort_flag, status);
      if (!ok) break;
      tc_fence_after();
      const uint64_t b0 = dv + ((sv * VTILE) >> 4);
      const uint32_t a0 = tmem + TM_SLOT0 + sl * 128;
      if (el) {
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          // P of keys 16k .. 16k+15 in columns 8k .. 8k+7 of the slot
          umma_ts_pair(tmem, a0 + 8 * k, b0 + ((k * 2048) >> 4), IDESC_PV2,
                       (j > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit_pair(&bar[PVDONE + sl], BOTH);
        umma_commit_pair(&bar[VEMPTY + sv], BOTH);
      }
      __syncwarp();
      // the slot's P is consumed (MMAs run in issue order): S(j + NSLOT)
      if (j + NSLOT < nblk) ok = issue_s(j + NSLOT);
    }
    if (ok && el) umma_commit_pair(&bar[OFINAL], BOTH);
    if (el) umma_commit_pair(&bar[DRAIN], BOTH);
    __syncwarp();
    wait_warp_drain(&bar[DRAIN], 0, status);
  } else if (kRopeQ && warp >= 10) {
    // ------------------------------------------------ Q rotation (RoPE) --
    const int tr = threadIdx.x - 320;  // 0..63
    if (wait_warp(&bar[QFULL], 0, abort_flag, status)) {
      for (int rr = tr; rr < RM; rr += 64)
        if (q0 + rr < args.Lq) rope_row(sQ, rr, q0 + rr, args);
      fence_proxy_async_smem();
      mbar_arrive(&bar[QREADY]);
    }
  } else if (warp < 8) {
    // ---------------------------------------------------------- softmax --
    setmaxnreg_inc();
    const int qd = warp & 3;
    const int h = warp >> 2;  // warp set: blocks j with j % 2 == h
    const int r = qd * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const float c2 = args.scale_log2;
    // keys this row may see: all kv_len, or its block-causal limit
    int row_lim = kv_len;
    if (args.chunk && q0 + r < args.Lq) {
      const int pos = q0 + r + args.q_offset;
      row_lim = min(args.Lk, (pos / args.chunk + 1) * args.chunk);
    }
    float m_w = -INFINITY;  // the max this warp last used
    float l_w = 0.f;        // this warp's row sum, relative to m_w
    bool ok = true;
    for (int j = h; j < nblk && ok; j += 2) {
      const int sl = j % NSLOT;
      ok = wait_warp(&bar[SFULL + sl], (j / NSLOT) & 1, abort_flag, status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_col = lane_base + TM_SLOT0 + sl * 128;
      float s[BN];
      tmem_ld128(s_col, s);
      tmem_ld_wait128(s);
      const int lim = row_lim - (kb0 + j) * BN;  // valid keys of this row
      const bool masked = __any_sync(0xffffffffu, lim < BN);
      if (masked) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      const float mx = (masked ? rowmax_masked<BN>(s) : rowmax<BN>(s)) * c2;
      // running max after block j: the previous block's, unless this block
      // exceeds it by more than 2^8 (p <= 256, exact after the final O / l)
      float m_prev = -INFINITY;
      if (j > 0) {
        ok = wait_warp(&bar[MCHAIN + qd], (j - 1) & 1, abort_flag, status);
        if (!ok) break;
        m_prev = s_mx[(j - 1) & 1][r];
      }
      const bool need = j > 0 && mx > m_prev + RESCALE_LOG2;
      const float m_j = (j == 0 || need) ? mx : m_prev;
      s_mx[j & 1][r] = m_j;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[MCHAIN + qd]);
      if (__any_sync(0xffffffffu, need)) {
        // O holds blocks 0 .. j-1 at m_prev once P V(j-1) has landed
        const float alpha = ex2(m_prev - m_j);
        ok = wait_warp(&bar[PVDONE + (j - 1) % NSLOT], ((j - 1) / NSLOT) & 1,
                       abort_flag, status);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(lane_base + c * 32, o);
          tmem_ld_wait32(o);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 v =
                ffma2(make_float2(o[e], o[e + 1]), make_float2(alpha, alpha),
                      make_float2(0.f, 0.f));
            o[e] = v.x;
            o[e + 1] = v.y;
          }
          tmem_st32(lane_base + c * 32, o);
        }
      }
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      // A row with no visible key yet (possible in a later key range) keeps
      // m = -inf: its scores are all -inf and exponentiate against 0 to
      // exact zeros.
      if (masked)
        exp_store_chunks<false>(s, c2, m_j == -INFINITY ? 0.f : m_j, s_col,
                                acc, 0, BN / 32);
      else
        exp_store_chunks<true, kPairEmu8>(s, c2, m_j, s_col, acc, 0,
                                          BN / 32);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (lead)
          mbar_arrive(&bar[PREADY + sl]);
        else
          mbar_arrive_remote_relaxed(
              mapa_shared(smem_u32(&bar[PREADY + sl]), 0));
      }
      const float2 tsum = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
      l_w = (m_w == m_j ? l_w : l_w * ex2(m_w - m_j)) + (tsum.x + tsum.y);
      m_w = m_j;
    }
    // the final max is the last block's; both sets' sums relative to it
    if (ok) ok = wait_warp(&bar[MCHAIN + qd], (nblk - 1) & 1, abort_flag,
                           status);
    if (ok) ok = wait_warp(&bar[OFINAL], 0, abort_flag, status);
    float m_fin = -INFINITY;
    if (ok) {
      m_fin = s_mx[(nblk - 1) & 1][r];
      s_xch[h][r] = m_w == -INFINITY ? 0.f : l_w * ex2(m_w - m_fin);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[XCH + qd]);
      ok = wait_warp(&bar[XCH + qd], 0, abort_flag, status);
    }
    if (ok) {
      tc_fence_after();
      const float l_tot = s_xch[0][r] + s_xch[1][r];
      // the item's coordinates again, rather than held through the loop
      int it_e = static_cast<int>(blockIdx.x >> 1);
      asm volatile("" : "+r"(it_e));
      const int split_e = it_e % args.n_split;
      it_e /= args.n_split;
      const int tx_e = it_e % args.n_tiles_x;
      const int head_e = (it_e / args.n_tiles_x) % args.heads;
      const int b_e = it_e / args.n_tiles_x / args.heads;
      const int tile_e = args.chunk ? args.n_tiles_x - 1 - tx_e : tx_e;
      const int row = tile_e * (2 * RM) + static_cast<int>(rank) * RM + r;
      const uint32_t o_col = lane_base + 64 * h;  // this set's 64 channels
      const int64_t orow_i =
          (static_cast<int64_t>(b_e) * args.Lq + row) * args.heads + head_e;
      if (args.n_split > 1) {
        // one key range of the row: unnormalised O (this set's channels)
        // and (row max, row sum) for the combining pass
        const int64_t prow = split_e * args.split_rows + orow_i;
        float4* dst =
            reinterpret_cast<float4*>(args.part_o + prow * HD + 64 * h);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float o[32];
          tmem_ld32(o_col + c * 32, o);
          tmem_ld_wait32(o);
          if (row < args.Lq) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[c * 8 + e] = make_float4(o[4 * e], o[4 * e + 1],
                                           o[4 * e + 2], o[4 * e + 3]);
          }
        }
        if (h == 0 && row < args.Lq)
          args.part_ml[prow] = make_float2(m_fin, l_tot);
      } else {
        const float inv = 1.0f / l_tot;
        __nv_bfloat16* orow = args.o + orow_i * HD + 64 * h;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float o[32];
          tmem_ld32(o_col + c * 32, o);
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
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA frees its memory while the pair's MMAs or the peer's
  // arrivals may still reach it
  cluster_sync_all();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Combining pass of a split key range: for each output row (b, token,
// head), the n_split partial results (unnormalised O_s, row max m_s in log2
// units, row sum l_s) give O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,
// M = max_s m_s -- the same online-softmax rescaling the kernel applies
// between key blocks.  One warp per row, 4 channels per lane.
__global__ void __launch_bounds__(256)
    combine_splits_kernel(const float4* __restrict__ part_o,
                          const float2* __restrict__ part_ml,
                          __nv_bfloat16* __restrict__ o, int64_t rows,
                          int n_split) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) +
                     (threadIdx.x >> 5);
       row < rows; row += warps) {
    float mmax = -INFINITY;
    for (int sp = 0; sp < n_split; ++sp)
      mmax = fmaxf(mmax, part_ml[sp * rows + row].x);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float l = 0.f;
    for (int sp = 0; sp < n_split; ++sp) {
      const float2 ml = part_ml[sp * rows + row];
      const float w = ml.x == -INFINITY ? 0.f : ex2(ml.x - mmax);
      const float4 v = part_o[(sp * rows + row) * (HD / 4) + lane];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
      l = fmaf(w, ml.y, l);
    }
    const float inv = 1.0f / l;
    uint2 out;
    out.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    out.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(o + row * HD)[lane] = out;
  }
}

// One warp waits, with the same bounded wait the attention kernel uses, on
// an mbarrier that needs one arrival and receives `arrive` (0 or 1).  With
// none the wait runs out after kWaitLimitNs, records WAN_ETIMEOUT in the
// device status word and the kernel returns: the timeout path can be
// checked without a fault or a hang.
__global__ void __launch_bounds__(32) wait_selftest_kernel(int arrive) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort;
  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (arrive && threadIdx.x == 0) mbar_arrive(&bar);
  __syncwarp();
  volatile int* abort_flag = &s_abort;
  wait_warp(&bar, 0, abort_flag, &g_wan_status);
}

// ------------------------------------------------------------------ host --

template <int kRope, int kPersist>
int launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
           const CUtensorMap& mo, AttnArgs a, int B, cudaStream_t s) {
  static std::mutex mu;
  static int state[64];  // 0 unknown, 1 ready, 2 unusable
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return WAN_ECUDA;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (state[dev] == 0) {
      // setmaxnreg draws on the registers the CTA was launched with: refuse
      // to launch if the compiled register count cannot fund the split
      // (the .inc would otherwise wait forever).
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, attn_fwd_kernel<kRope, kPersist>) !=
          cudaSuccess)
        return WAN_ECUDA;
      const int need = 8 * 32 * kSoftmaxRegs + 4 * 32 * kOtherRegs;
      if (fa.numRegs * kThreads < need) {
        state[dev] = 2;
      } else if (cudaFuncSetAttribute(
                     attn_fwd_kernel<kRope, kPersist>,
                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                     SMEM_DYN) != cudaSuccess) {
        return WAN_ECUDA;
      } else {
        state[dev] = 1;
      }
    }
    if (state[dev] != 1) return WAN_EUNSUPPORTED;
  }
  a.n_tiles_x = (a.Lq + QT * BM - 1) / (QT * BM);
  const int64_t items =
      static_cast<int64_t>(a.n_tiles_x) * a.heads * B * a.n_split;
  if (items > INT32_MAX) return WAN_EINVAL;
  a.items = static_cast<int>(items);
  // One CTA per item, except cross-attention: its items are short (a few
  // key blocks), so one persistent CTA per SM walks them and loads the next
  // item's Q while the current one drains.
  int grid = a.items;
  if (kPersist) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
        cudaSuccess)
      return WAN_ECUDA;
    grid = a.items < sms ? a.items : sms;
  }
  attn_fwd_kernel<kRope, kPersist><<<grid, kThreads, SMEM_DYN, s>>>(
      mq, mk, mv, mo, a);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}

template <int kRopeQ>
int launch_pair(const CUtensorMap& mq, const CUtensorMap& mk,
                const CUtensorMap& mv, AttnArgs a, int B, cudaStream_t s) {
  static std::mutex mu;
  static int state[64];  // 0 unknown, 1 ready
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return WAN_ECUDA;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (state[dev] == 0) {
      // setmaxnreg draws on the registers the CTA was launched with
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, attn_pair_kernel<kRopeQ>) != cudaSuccess)
        return WAN_ECUDA;
      if (fa.numRegs * pair::THREADS <
          8 * 32 * kSoftmaxRegs + 4 * 32 * kOtherRegs)
        return WAN_EUNSUPPORTED;
      if (cudaFuncSetAttribute(attn_pair_kernel<kRopeQ>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               pair::SMEM) != cudaSuccess)
        return WAN_ECUDA;
      state[dev] = 1;
    }
  }
  a.n_tiles_x = (a.Lq + 2 * pair::RM - 1) / (2 * pair::RM);
  const int64_t items =
      static_cast<int64_t>(a.n_tiles_x) * a.heads * B * a.n_split;
  if (2 * items > INT32_MAX) return WAN_EINVAL;
  a.items = static_cast<int>(items);
  attn_pair_kernel<kRopeQ><<<static_cast<unsigned>(2 * items), pair::THREADS,
                             pair::SMEM, s>>>(mq, mk, mv, a);
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


// Key limit of the last query row of two-tile item `tile` (block-causal).
int causal_item_kv(int tile, int Lq, int Lk, int chunk, int q_offset) {
  const int last = min((tile + 1) * QT * BM, Lq) - 1 + q_offset;
  return min(Lk, (last / chunk + 1) * chunk);
}

// Key ranges for `items` equal work items of nblk key blocks on `slots`
// concurrent CTAs (or CTA pairs): the smallest count up to 4, with at least
// 8 key blocks a range, whose waves are at least 95 % full (else the
// fullest).  range_cost discounts a split count's wave fill by the
// measured cost of its fp32 partials and combining pass.
int split_count(double items, int nblk, int slots, double range_cost) {
  int best = 1;
  double best_eff = 0.0;
  for (int sp = 1; sp <= 4; ++sp) {
    if (sp > 1 && nblk < 8 * sp) break;  // at least 8 key blocks per range
    const double waves = items * sp / slots;
    const double eff = waves / ceil(waves) * (sp > 1 ? 1.0 - range_cost : 1.0);
    if (eff > best_eff + 0.01) {
      best = sp;
      best_eff = eff;
    }
    if (eff >= 0.95) break;
  }
  return best;
}

// Rows of partial results and the combining pass of a split call.
int combine_splits(const AttnArgs& a, int64_t rows, int n_split,
                   cudaStream_t cs) {
  const int64_t blocks64 = (rows + 7) / 8;
  const int blocks =
      static_cast<int>(blocks64 < 148 * 16 ? blocks64 : 148 * 16);
  combine_splits_kernel<<<blocks, 256, 0, cs>>>(
      reinterpret_cast<const float4*>(a.part_o), a.part_ml, a.o, rows,
      n_split);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
}

int causal_check(const void* q, const void* k, const void* v, void* o, int B,
                 int Lq, int Lk, int heads, int head_dim, int chunk_tokens,
                 int q_offset, float softmax_scale) {
  int st = check_common(q, k, v, o, B, Lq, Lk, heads, head_dim,
                        softmax_scale);
  if (st != WAN_OK) return st;
  if (chunk_tokens < 1 || q_offset < 0 ||
      static_cast<int64_t>(q_offset) + Lq > Lk)
    return WAN_EINVAL;
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
  if ((st = make_map_bf16(&mq, q, B, L, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mk, k, B, L, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mv, v, B, L, heads, BM)) != WAN_OK) return st;
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
  a.chunk = 0;
  a.q_offset = 0;
  CUtensorMap mo;
  if ((st = make_map_bf16(&mo, o, B, a.Lq, heads, BM)) != WAN_OK)
    return st;
  return d_table ? launch<1, 0>(mq, mk, mv, mo, a, B, as_stream(s))
                 : launch<0, 0>(mq, mk, mv, mo, a, B, as_stream(s));
}

int wan_self_attn_rope_q(const void* q, const void* k, const void* v,
                         void* o, int B, wan_grid_t g, int heads,
                         int head_dim, const void* d_table,
                         float softmax_scale, void* s) {
  using namespace wan;
  if (!d_table) return WAN_EINVAL;
  if (g.F < 1 || g.H < 1 || g.W < 1) return WAN_EINVAL;
  const int64_t L64 = static_cast<int64_t>(g.F) * g.H * g.W;
  if (L64 > (1 << 26)) return WAN_EINVAL;
  const int L = static_cast<int>(L64);
  int st = check_common(q, k, v, o, B, L, L, heads, head_dim, softmax_scale);
  if (st != WAN_OK) return st;
  if (wan_rope3d_table_bytes(g, head_dim) == 0) return WAN_EINVAL;
  if (!aligned16(d_table)) return WAN_EALIGN;
  st = check_device(nullptr);
  if (st != WAN_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map_bf16(&mq, q, B, L, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mk, k, B, L, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mv, v, B, L, heads, BM)) != WAN_OK) return st;
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
  a.chunk = 0;
  a.q_offset = 0;
  CUtensorMap mo;
  if ((st = make_map_bf16(&mo, o, B, a.Lq, heads, BM)) != WAN_OK)
    return st;
  return launch<2, 0>(mq, mk, mv, mo, a, B, as_stream(s));
}

int wan_self_attn_pair(const void* q, const void* k, const void* v, void* o,
                       int B, wan_grid_t g, int heads, int head_dim,
                       const void* d_table_q, float softmax_scale, void* s) {
  using namespace wan;
  if (g.F < 1 || g.H < 1 || g.W < 1) return WAN_EINVAL;
  const int64_t L64 = static_cast<int64_t>(g.F) * g.H * g.W;
  if (L64 > (1 << 26)) return WAN_EINVAL;
  const int L = static_cast<int>(L64);
  int st = check_common(q, k, v, o, B, L, L, heads, head_dim, softmax_scale);
  if (st != WAN_OK) return st;
  if (d_table_q) {
    if (wan_rope3d_table_bytes(g, head_dim) == 0) return WAN_EINVAL;
    if (!aligned16(d_table_q)) return WAN_EALIGN;
  }
  st = check_device(nullptr);
  if (st != WAN_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map_bf16(&mq, q, B, L, heads, 128)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mk, k, B, L, heads, 64)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mv, v, B, L, heads, 128)) != WAN_OK) return st;
  AttnArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.table = static_cast<const float4*>(d_table_q);
  a.Lq = L;
  a.Lk = L;
  a.heads = heads;
  a.F = g.F;
  a.H = g.H;
  a.W = g.W;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.cross = 0;
  a.chunk = 0;
  a.q_offset = 0;
  return d_table_q ? launch_pair<1>(mq, mk, mv, a, B, as_stream(s))
                   : launch_pair<0>(mq, mk, mv, a, B, as_stream(s));
}


size_t wan_block_causal_attn_workspace_bytes(int B, int Lq, int heads,
                                             int n_split) {
  if (B < 1 || Lq < 1 || heads < 1 || n_split < 1 || n_split > 8) return 0;
  if (n_split == 1) return 0;
  return static_cast<size_t>(n_split) * B * Lq * heads *
         (wan::HD * sizeof(float) + 2 * sizeof(float));
}

int wan_block_causal_attn_splits(int B, int Lq, int Lk, int heads,
                                 int chunk_tokens, int q_offset) {
  using namespace wan;
  if (B < 1 || Lq < 1 || Lk < 1 || heads < 1 || chunk_tokens < 1 ||
      q_offset < 0 || static_cast<int64_t>(q_offset) + Lq > Lk)
    return WAN_EINVAL;
  int dev = 0;
  int st = check_device(&dev);
  if (st != WAN_OK) return st;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess)
    return WAN_ECUDA;
  const int tiles = (Lq + QT * BM - 1) / (QT * BM);
  const int kv_first = causal_item_kv(0, Lq, Lk, chunk_tokens, q_offset);
  const int kv_last =
      causal_item_kv(tiles - 1, Lq, Lk, chunk_tokens, q_offset);
  // Unequal items already run heaviest first; equal ones (a KV-cache step,
  // where every query sees the whole cache) are split when their count
  // leaves the last wave of CTAs partly empty.
  if (kv_first != kv_last) return 1;
  const int nblk = (kv_first + BN - 1) / BN;
  return split_count(static_cast<double>(tiles) * heads * B, nblk, sms, 0.0);
}

int wan_block_causal_attn_split(const void* q, const void* k, const void* v,
                                void* o, int B, int Lq, int Lk, int heads,
                                int head_dim, int chunk_tokens, int q_offset,
                                float softmax_scale, int n_split,
                                void* workspace, size_t workspace_bytes,
                                void* s) {
  using namespace wan;
  int st = causal_check(q, k, v, o, B, Lq, Lk, heads, head_dim, chunk_tokens,
                        q_offset, softmax_scale);
  if (st != WAN_OK) return st;
  if (n_split < 1 || n_split > 8) return WAN_EINVAL;
  if (n_split > 1) {
    // every key range of every item holds at least one key block
    const int kv0 = causal_item_kv(0, Lq, Lk, chunk_tokens, q_offset);
    if ((kv0 + BN - 1) / BN < n_split) return WAN_EINVAL;
    const size_t need =
        wan_block_causal_attn_workspace_bytes(B, Lq, heads, n_split);
    if (!workspace || workspace_bytes < need) return WAN_EINVAL;
    if (!aligned16(workspace)) return WAN_EALIGN;
  }
  st = check_device(nullptr);
  if (st != WAN_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map_bf16(&mq, q, B, Lq, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mk, k, B, Lk, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mv, v, B, Lk, heads, BM)) != WAN_OK) return st;
  AttnArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.table = nullptr;
  a.Lq = Lq;
  a.Lk = Lk;
  a.heads = heads;
  a.F = a.H = a.W = 1;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.cross = 0;
  a.chunk = chunk_tokens;
  a.q_offset = q_offset;
  a.n_split = n_split;
  const int64_t rows = static_cast<int64_t>(B) * Lq * heads;
  if (n_split > 1) {
    a.part_o = static_cast<float*>(workspace);
    a.part_ml = reinterpret_cast<float2*>(a.part_o + n_split * rows * HD);
    a.split_rows = rows;
  }
  cudaStream_t cs = as_stream(s);
  CUtensorMap mo;
  if ((st = make_map_bf16(&mo, o, B, a.Lq, heads, BM)) != WAN_OK)
    return st;
  st = launch<0, 0>(mq, mk, mv, mo, a, B, cs);
  if (st != WAN_OK || n_split == 1) return st;
  return combine_splits(a, rows, n_split, cs);
}

// ------------------------------------------------- without allocation --
// Scratch of wan_block_causal_attn_split_noalloc: a fixed array in device
// memory, created when the library is loaded on a device and held until the
// process exits, so that the call needs no allocation.  Shared by every
// call on that device.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[kNoAllocScratchBytes];

int wan_block_causal_attn_split_noalloc(const void* q, const void* k,
                                        const void* v, void* o, int B, int Lq,
                                        int Lk, int heads, int head_dim,
                                        int chunk_tokens, int q_offset,
                                        float softmax_scale, int n_split,
                                        void* s) {
  const size_t need =
      wan_block_causal_attn_workspace_bytes(B, Lq, heads, n_split);
  if (n_split > 1 && need == 0) return WAN_EINVAL;
  if (need > kNoAllocScratchBytes) return WAN_ENOSPACE;
  int dev = 0;
  int st = wan::check_device(&dev);
  if (st != WAN_OK) return st;
  // Device address of the scratch array on this device: looked up once per
  // device, with that device current (in host code the array's name is
  // only a stand-in for it).
  static std::mutex mu;
  static void* addr[64];
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess ||
          !ptr)
        return WAN_ECUDA;
      addr[dev] = ptr;
    }
    ws = addr[dev];
  }
  return wan_block_causal_attn_split(q, k, v, o, B, Lq, Lk, heads, head_dim,
                                     chunk_tokens, q_offset, softmax_scale,
                                     n_split, n_split > 1 ? ws : nullptr,
                                     n_split > 1 ? kNoAllocScratchBytes : 0,
                                     s);
}

size_t wan_block_causal_attn_noalloc_max_bytes(void) {
  return kNoAllocScratchBytes;
}

int wan_attn_pair_resident_clusters(void) {
  using namespace wan;
  int st = check_device(nullptr);
  if (st != WAN_OK) return st;
  if (cudaFuncSetAttribute(attn_pair_kernel<0>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           pair::SMEM) != cudaSuccess)
    return WAN_ECUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(pair::THREADS, 1, 1);
  cfg.dynamicSmemBytes = pair::SMEM;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, attn_pair_kernel<0>, &cfg) !=
      cudaSuccess)
    return WAN_ECUDA;
  return n;
}

int wan_block_causal_attn_pair(const void* q, const void* k, const void* v,
                               void* o, int B, int Lq, int Lk, int heads,
                               int head_dim, int chunk_tokens, int q_offset,
                               float softmax_scale, void* s) {
  using namespace wan;
  int st = check_common(q, k, v, o, B, Lq, Lk, heads, head_dim,
                        softmax_scale);
  if (st != WAN_OK) return st;
  if (chunk_tokens < 1 || q_offset < 0 ||
      static_cast<int64_t>(q_offset) + Lq > Lk)
    return WAN_EINVAL;
  st = check_device(nullptr);
  if (st != WAN_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map_bf16(&mq, q, B, Lq, heads, 128)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mk, k, B, Lk, heads, 64)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mv, v, B, Lk, heads, 128)) != WAN_OK) return st;
  AttnArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.table = nullptr;
  a.Lq = Lq;
  a.Lk = Lk;
  a.heads = heads;
  a.F = a.H = a.W = 1;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.cross = 0;
  a.chunk = chunk_tokens;
  a.q_offset = q_offset;
  return launch_pair<0>(mq, mk, mv, a, B, as_stream(s));
}

int wan_block_causal_attn_pair_splits(int B, int Lq, int Lk, int heads,
                                      int chunk_tokens, int q_offset) {
  using namespace wan;
  if (B < 1 || Lq < 1 || Lk < 1 || heads < 1 || chunk_tokens < 1 ||
      q_offset < 0 || static_cast<int64_t>(q_offset) + Lq > Lk)
    return WAN_EINVAL;
  const int pairs = wan_attn_pair_resident_clusters();
  if (pairs < 1) return pairs < 0 ? pairs : WAN_EUNSUPPORTED;
  // pair items hold 256 query rows, as the two-tile kernel's do
  const int tiles = (Lq + 2 * pair::RM - 1) / (2 * pair::RM);
  const int kv_first = causal_item_kv(0, Lq, Lk, chunk_tokens, q_offset);
  const int kv_last =
      causal_item_kv(tiles - 1, Lq, Lk, chunk_tokens, q_offset);
  if (kv_first != kv_last) return 1;
  const int nblk = (kv_first + BN - 1) / BN;
  // Measured at the 480p-165f KV-cache step (760 pair items on 74 pairs):
  // 2 ranges (waves 97.8 % full) ran 1.3 % slower than one (93.4 %), so a
  // split must buy more than about 6 % of wave fill.
  return split_count(static_cast<double>(tiles) * heads * B, nblk, pairs,
                     0.06);
}

int wan_block_causal_attn_pair_split(const void* q, const void* k,
                                     const void* v, void* o, int B, int Lq,
                                     int Lk, int heads, int head_dim,
                                     int chunk_tokens, int q_offset,
                                     float softmax_scale, int n_split,
                                     void* workspace, size_t workspace_bytes,
                                     void* s) {
  using namespace wan;
  int st = causal_check(q, k, v, o, B, Lq, Lk, heads, head_dim, chunk_tokens,
                        q_offset, softmax_scale);
  if (st != WAN_OK) return st;
  if (n_split < 1 || n_split > 8) return WAN_EINVAL;
  if (n_split > 1) {
    // every key range of every item holds at least one key block
    const int kv0 = causal_item_kv(0, Lq, Lk, chunk_tokens, q_offset);
    if ((kv0 + BN - 1) / BN < n_split) return WAN_EINVAL;
    const size_t need =
        wan_block_causal_attn_workspace_bytes(B, Lq, heads, n_split);
    if (!workspace || workspace_bytes < need) return WAN_EINVAL;
    if (!aligned16(workspace)) return WAN_EALIGN;
  }
  st = check_device(nullptr);
  if (st != WAN_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map_bf16(&mq, q, B, Lq, heads, 128)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mk, k, B, Lk, heads, 64)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mv, v, B, Lk, heads, 128)) != WAN_OK) return st;
  AttnArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.table = nullptr;
  a.Lq = Lq;
  a.Lk = Lk;
  a.heads = heads;
  a.F = a.H = a.W = 1;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.cross = 0;
  a.chunk = chunk_tokens;
  a.q_offset = q_offset;
  a.n_split = n_split;
  const int64_t rows = static_cast<int64_t>(B) * Lq * heads;
  if (n_split > 1) {
    a.part_o = static_cast<float*>(workspace);
    a.part_ml = reinterpret_cast<float2*>(a.part_o + n_split * rows * HD);
    a.split_rows = rows;
  }
  cudaStream_t cs = as_stream(s);
  st = launch_pair<0>(mq, mk, mv, a, B, cs);
  if (st != WAN_OK || n_split == 1) return st;
  return combine_splits(a, rows, n_split, cs);
}

int wan_block_causal_attn(const void* q, const void* k, const void* v,
                          void* o, int B, int Lq, int Lk, int heads,
                          int head_dim, int chunk_tokens, int q_offset,
                          float softmax_scale, void* s) {
  using namespace wan;
  int st = check_common(q, k, v, o, B, Lq, Lk, heads, head_dim,
                        softmax_scale);
  if (st != WAN_OK) return st;
  if (chunk_tokens < 1 || q_offset < 0 ||
      static_cast<int64_t>(q_offset) + Lq > Lk)
    return WAN_EINVAL;
  st = check_device(nullptr);
  if (st != WAN_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map_bf16(&mq, q, B, Lq, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mk, k, B, Lk, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mv, v, B, Lk, heads, BM)) != WAN_OK) return st;
  AttnArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.table = nullptr;
  a.Lq = Lq;
  a.Lk = Lk;
  a.heads = heads;
  a.F = a.H = a.W = 1;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.cross = 0;
  a.chunk = chunk_tokens;
  a.q_offset = q_offset;
  CUtensorMap mo;
  if ((st = make_map_bf16(&mo, o, B, a.Lq, heads, BM)) != WAN_OK)
    return st;
  return launch<0, 0>(mq, mk, mv, mo, a, B, as_stream(s));
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
  if ((st = make_map_bf16(&mq, q, B, Lq, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mk, k_ctx, B, Lk, heads, BM)) != WAN_OK) return st;
  if ((st = make_map_bf16(&mv, v_ctx, B, Lk, heads, BM)) != WAN_OK) return st;
  AttnArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.table = nullptr;
  a.Lq = Lq;
  a.Lk = Lk;
  a.heads = heads;
  a.F = a.H = a.W = 1;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.cross = 1;
  a.chunk = 0;
  a.q_offset = 0;
  for (int i = 0; i < B; ++i) a.lens[i] = ctx_lens[i];
  CUtensorMap mo;
  if ((st = make_map_bf16(&mo, o, B, Lq, heads, BM)) != WAN_OK) return st;
  return launch<0, 1>(mq, mk, mv, mo, a, B, as_stream(s));
}

int wan_wait_selftest(int arrive, void* s) {
  if (arrive != 0 && arrive != 1) return WAN_EINVAL;
  int st = wan::check_device(nullptr);
  if (st != WAN_OK) return st;
  wan::wait_selftest_kernel<<<1, 32, 0, wan::as_stream(s)>>>(arrive);
  return cudaGetLastError() == cudaSuccess ? WAN_OK : WAN_ECUDA;
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
