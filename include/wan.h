/*
 * wan.h -- C ABI of libwan, the B200 (sm_100a) hot path of the Wan2.1 /
 * Wan2.2 video diffusion transformer: 3D RoPE, full spatio-temporal
 * self-attention, length-masked cross-attention to text, block-causal
 * (chunked, KV-cache) attention, the block prologue / epilogue (AdaLN
 * modulate, QK-Norm + RoPE, gated residual), the shifted sigma schedule
 * with the fused CFG + Euler flow step, the fused UniPC order-2 sampler
 * stop, and the layout moves around the Ulysses all-to-all.
 *
 * Sources (cited by page and section):
 *   "Wan2.2 source reading" -- blog.leeguoo.com, "動画生成の勘定を明らかにする：
 *       Wan2.2 ソースコード精読";
 *   "Wan paper explainer"   -- 0h-n0.github.io, "論文解説: Wan - 大規模オープン
 *       ソース動画生成モデルのアーキテクチャと訓練";
 *   "Long-video survey"     -- the atlascloud.ai long-video generation blog.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Attention tensors are bf16, contiguous, row-major [B, L, heads, head_dim]
 *   (token-major, heads interleaved: the natural layout of a [B, L, dim]
 *   projection with dim = heads * head_dim).  head_dim must be 128.
 * - Token order inside L is frame-major: n = (f * H + h) * W + w.
 * - Device pointers are plain CUDA device addresses owned by the caller; the
 *   library allocates no device memory and keeps no per-call state.  Every
 *   launch goes to the caller's stream `s` (a cudaStream_t passed as void*,
 *   NULL = legacy default stream).  No call synchronises the stream.
 * - Return values: WAN_OK (0) or a negative wan_status.  Argument checks are
 *   synchronous and leave the device untouched.  A failed launch returns
 *   WAN_ECUDA.  Device-side faults surface at the caller's next synchronise.
 * - Every wait inside a kernel is bounded (about two seconds); a wait that
 *   runs out records WAN_ETIMEOUT in a device status word, read and cleared
 *   by wan_device_status().
 */
#ifndef WAN_H_
#define WAN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Token grid after the (1, 2, 2) patchify: L = F * H * W. */
typedef struct {
  int32_t F, H, W;
} wan_grid_t;

enum wan_status {
  WAN_OK = 0,
  WAN_EINVAL = -1,        /* bad size, null pointer, out-of-range value   */
  WAN_EALIGN = -2,        /* pointer not 16-byte aligned                   */
  WAN_EUNSUPPORTED = -3,  /* current device is not sm_100 (B200 class)     */
  WAN_ECUDA = -4,         /* a CUDA runtime call or launch failed          */
  WAN_ETIMEOUT = -5,      /* a bounded in-kernel wait ran out              */
  WAN_ENOSPACE = -6       /* needs more scratch than the library's fixed
                             array holds (the no-allocation call)          */
};

/* Static text of a status code (never NULL). */
const char* wan_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int wan_version(void);

/* ---------------------------------------------------------------- grid --
 * Wan2.2 source reading, ch. 2 "VAE" (target_shape, vae_stride (4, 8, 8),
 * frames of the form 4n+1) and ch. 4 "From latent to token" (patch (1,2,2)).
 * Host only.  frames = 4n+1 >= 1, height and width multiples of 16 (8 for
 * the VAE times 2 for the patch).  Writes the latent shape
 * (16, (frames-1)/4+1, height/8, width/8) to latent_out[4] if it is not NULL
 * and the token grid to *grid_out.  Returns WAN_EINVAL otherwise.          */
int wan_token_grid(int frames, int height, int width, int32_t* latent_out,
                   wan_grid_t* grid_out);

/* ---------------------------------------------------------------- RoPE --
 * Wan2.2 source reading, ch. 4, section "3D RoPE": per head the 128
 * channels split into a time band of 44 and height / width bands of 42
 * (concatenated t, h, w); adjacent channels (2j, 2j+1) form one complex
 * number that is turned by pos * theta^(-2j / D_band), pos being the
 * token's f, h or w coordinate; the page rotates in float64.
 *
 * Table layout (float2 = {cos, sin}, fp32, computed in fp64 on the host):
 *   rows 0 .. F-1        : time band,   entry e = j        (j = 0..21)
 *   rows F .. F+H-1      : height band, entry e = j        (j = 0..20), e=21 pad
 *   rows F+H .. F+H+W-1  : width band,  entry e = j + 1    (j = 0..20), e=0 pad
 * every row has 22 entries (176 bytes), pads hold {1, 0}.  With this layout
 * the absolute pair index p = 2m, 2m+1 of a 16-byte load always lands on a
 * 16-byte aligned table address.
 *
 * wan_rope3d_table_bytes: size of that table.  Returns 0 for a bad grid.
 * wan_rope3d_table: fills caller-owned device memory d_table (bytes >= the
 *   size above) with an asynchronous copy from a library-held host staging
 *   buffer on stream s.  grid sides must be in 1..1024 (the page builds the
 *   tables for 1024 positions), head_dim 128, theta > 0.  Not capturable in a
 *   CUDA graph (pageable host copy).
 * wan_rope3d_qk: rotates q and k in place (bf16 in, fp32 arithmetic, bf16
 *   out), [B, L, heads, 128] with L = F*H*W, using the table above.  q or k
 *   may be NULL to rotate only the other.                                   */
size_t wan_rope3d_table_bytes(wan_grid_t g, int head_dim);
int wan_rope3d_table(wan_grid_t g, int head_dim, double theta, void* d_table,
                     size_t bytes, void* s);
int wan_rope3d_qk(void* q, void* k, int B, wan_grid_t g, int heads,
                  int head_dim, const void* d_table, void* s);

/* ------------------------------------------------------- self-attention --
 * Wan2.2 source reading, ch. 4 "Full forward of one block" and ch. 8 "What
 * is 75600^2": full bidirectional attention over all L = F*H*W tokens,
 *   O = softmax(Q K^T * softmax_scale) V,   no mask.
 * q, k, v, o: [B, L, heads, 128] bf16, 16-byte aligned; o must not alias
 * q, k or v.  If d_table is not NULL (the table above for grid g), Q and K
 * are rotated by the 3D RoPE inside the kernel as their tiles are staged
 * (q and k in memory are left untouched); if NULL, q and k are used as given
 * (already rotated, e.g. by wan_rope3d_qk).  fp32 accumulation and softmax,
 * bf16 output.  softmax_scale > 0 (the pages use 1/sqrt(head_dim)).        */
int wan_self_attn(const void* q, const void* k, const void* v, void* o,
                  int B, wan_grid_t g, int heads, int head_dim,
                  const void* d_table, float softmax_scale, void* s);

/* Self-attention with q rotated by the 3D RoPE in the attention kernel's
 * tile stage (once per 256-row query tile, in shared memory; q in memory is
 * untouched) and k already rotated -- e.g. by wan_rope3d_qk with a NULL q,
 * or by wan_qk_norm_rope, which writes the rotated k anyway.  Rotating k in
 * the tile stage (wan_self_attn with a table) repeats the rotation of every
 * key block in every query tile; this form rotates each key once.  d_table
 * is required.  Otherwise the same layouts, arguments, errors and results
 * as wan_self_attn.  Source: Wan2.2 source reading, ch. 4 "3D RoPE".       */
int wan_self_attn_rope_q(const void* q, const void* k, const void* v,
                         void* o, int B, wan_grid_t g, int heads,
                         int head_dim, const void* d_table,
                         float softmax_scale, void* s);

/* The same full self-attention computed by pairs of CTAs on two SMs: one
 * tcgen05 MMA (cta_group::2) covers 256 query rows, 128 in each SM's tensor
 * memory, with each SM staging half of every K / V block; three score slots
 * per SM let the Q K^T of later blocks run while the softmax of an earlier
 * one is still going.  k must already be rotated (wan_rope3d_qk with a NULL
 * q rotates k alone).  If d_table_q is NULL, q is used as given (already
 * rotated); otherwise q is rotated by the 3D RoPE in shared memory, once per
 * query tile, before the tensor cores read it (q in memory is untouched).
 * Otherwise the same layouts, arguments, errors and results as
 * wan_self_attn.  Source: Wan2.2 source reading, ch. 4 "Full forward of one
 * block", "3D RoPE" and ch. 8.                                             */
int wan_self_attn_pair(const void* q, const void* k, const void* v, void* o,
                       int B, wan_grid_t g, int heads, int head_dim,
                       const void* d_table_q, float softmax_scale, void* s);

/* ------------------------------------------------------ cross-attention --
 * Wan2.2 source reading, ch. 3 "Where did the prompt go" (each prompt is
 * trimmed to its true length; video tokens query, the text context is
 * key/value) and Wan paper explainer, section "Text encoder"
 * (softmax(Q K_text^T / sqrt(d_k)) V_text):
 *   O[b] = softmax(Q[b] K_ctx[b, :len_b]^T * softmax_scale) V_ctx[b, :len_b]
 * q, o: [B, Lq, heads, 128]; k_ctx, v_ctx: [B, Lk, heads, 128] bf16.
 * ctx_lens: HOST array of B int32 with 1 <= len_b <= Lk; it is read during
 * the call.  Rows j >= len_b of k_ctx / v_ctx are never used, whatever they
 * hold (NaN included).  No RoPE.  B <= 512.                               */
int wan_cross_attn(const void* q, const void* k_ctx, const void* v_ctx,
                   void* o, const int32_t* ctx_lens, int B, int Lq, int Lk,
                   int heads, int head_dim, float softmax_scale, void* s);

/* ------------------------------------------------ block-causal (chunks) --
 * Long-video survey (atlascloud.ai), section "Route 3 · Self Forcing":
 * bidirectional attention is replaced by causal attention over chunks of
 * frames, each chunk attending to earlier chunks through a KV cache.  A
 * query at absolute token position a = q_offset + i sees keys
 *   j < min(Lk, (floor(a / chunk_tokens) + 1) * chunk_tokens),
 * i.e. its own chunk and all earlier ones:
 *   O = softmax(Q K^T * softmax_scale + mask) V.
 * Full sequence: q_offset = 0, Lq = Lk.  KV-cache step: the queries of one
 * chunk (Lq tokens at absolute positions q_offset ..) against the cached
 * keys followed by that chunk (Lk >= q_offset + Lq).  q, o: [B, Lq, heads,
 * 128]; k, v: [B, Lk, heads, 128] bf16, already rotated (wan_rope3d_qk).
 * chunk_tokens >= 1, q_offset >= 0, q_offset + Lq <= Lk.  Keys beyond a
 * row's limit get weight exactly 0; as they can share a key block with
 * visible keys they must be finite (0 * NaN would not vanish).             */
int wan_block_causal_attn(const void* q, const void* k, const void* v,
                          void* o, int B, int Lq, int Lk, int heads,
                          int head_dim, int chunk_tokens, int q_offset,
                          float softmax_scale, void* s);

/* The same block-causal attention with each (256-row tile, head, batch row)
 * work item's key blocks cut into n_split consecutive ranges run as separate
 * CTAs, followed by a combining pass.  When every query of the call sees the
 * same keys (a KV-cache step over the whole cache) the items are equal, and
 * their count can leave the last wave of CTAs mostly idle (760 items on 148
 * SMs is 5.1 waves); n_split ranges make n_split times as many shorter
 * items.  Each range writes its rows' unnormalised fp32 O and (row max, row
 * sum) into `workspace`; the combining pass rescales and sums them, the
 * online-softmax step of the kernel applied across ranges, and writes bf16
 * o.  The result equals wan_block_causal_attn's up to fp32 summation order.
 * n_split in [1, 8] and at most the key-block count of the lightest item
 * (WAN_EINVAL otherwise); n_split == 1 is wan_block_causal_attn.
 * workspace: caller-owned device memory of at least
 * wan_block_causal_attn_workspace_bytes(B, Lq, heads, n_split) bytes,
 * 16-byte aligned (NULL allowed when that is 0); its contents on entry do
 * not matter and on return are unspecified.  Calls that share a workspace
 * must not overlap on the device.                                         */
int wan_block_causal_attn_split(const void* q, const void* k, const void* v,
                                void* o, int B, int Lq, int Lk, int heads,
                                int head_dim, int chunk_tokens, int q_offset,
                                float softmax_scale, int n_split,
                                void* workspace, size_t workspace_bytes,
                                void* s);

/* Workspace bytes of wan_block_causal_attn_split: n_split * B * Lq * heads
 * * (128 * 4 + 8) for n_split > 1, 0 for n_split == 1 or bad arguments.    */
size_t wan_block_causal_attn_workspace_bytes(int B, int Lq, int heads,
                                             int n_split);

/* Host: the key-range count wan_block_causal_attn_split is fastest with on
 * the current device: 1 unless every item sees the same keys; otherwise the
 * smallest count (up to 4, at least 8 key blocks per range) whose waves of
 * CTAs are at least 95 % full, else the fullest.  Negative wan_status on
 * bad arguments.                                                           */
int wan_block_causal_attn_splits(int B, int Lq, int Lk, int heads,
                                 int chunk_tokens, int q_offset);

/* wan_block_causal_attn_split for callers that cannot allocate device
 * memory: the pages have no counterpart of this call.  Some callers must
 * not allocate once they run -- a serving loop whose memory is fixed at
 * start-up (an allocation can synchronise the device and stall the other
 * streams), or code embedded in a host application that owns all device
 * memory and offers no allocator -- and so cannot provide the workspace.
 * This call takes its scratch from a fixed array in device memory instead:
 * 64 MiB (wan_block_causal_attn_noalloc_max_bytes()), created on each GPU
 * that loads the library and held until the process exits.  Calls whose
 * wan_block_causal_attn_workspace_bytes(B, Lq, heads, n_split) exceeds it
 * return WAN_ENOSPACE without touching the device.  The first call on a
 * device looks up the array's device address (with that device current)
 * and keeps it; make that first call before any stream capture.  Every
 * call on a device shares the one array, and it keeps the last call's
 * contents; nothing in it needs to start at zero (each call writes every
 * value it reads).  Calls that overlap on the GPU -- on different streams,
 * or from different host threads -- race on the array and give wrong
 * results; serialise them.  Arguments, results and other errors as
 * wan_block_causal_attn_split, without the workspace arguments.           */
int wan_block_causal_attn_split_noalloc(const void* q, const void* k,
                                        const void* v, void* o, int B, int Lq,
                                        int Lk, int heads, int head_dim,
                                        int chunk_tokens, int q_offset,
                                        float softmax_scale, int n_split,
                                        void* s);

/* Bytes of the fixed scratch array of wan_block_causal_attn_split_noalloc. */
size_t wan_block_causal_attn_noalloc_max_bytes(void);

/* The same block-causal attention computed by pairs of CTAs on two SMs (the
 * kernel of wan_self_attn_pair, with the per-row key limit above; the
 * 256-row tiles of each head run heaviest first).  Same arguments, layouts,
 * errors and results as wan_block_causal_attn.                            */
int wan_block_causal_attn_pair(const void* q, const void* k, const void* v,
                               void* o, int B, int Lq, int Lk, int heads,
                               int head_dim, int chunk_tokens, int q_offset,
                               float softmax_scale, void* s);

/* wan_block_causal_attn_split on the CTA-pair kernel: each (256-row tile,
 * head, batch row) pair item's key blocks cut into n_split consecutive
 * ranges run as separate CTA pairs, then the same combining pass.  The
 * workspace has the size and layout of wan_block_causal_attn_split's
 * (wan_block_causal_attn_workspace_bytes); arguments, errors and results
 * are those of wan_block_causal_attn_split.                                */
int wan_block_causal_attn_pair_split(const void* q, const void* k,
                                     const void* v, void* o, int B, int Lq,
                                     int Lk, int heads, int head_dim,
                                     int chunk_tokens, int q_offset,
                                     float softmax_scale, int n_split,
                                     void* workspace, size_t workspace_bytes,
                                     void* s);

/* Key-range count for wan_block_causal_attn_pair_split: 1 unless every
 * item sees the same keys; otherwise the count up to 4 (at least 8 key
 * blocks a range) whose waves of CTA pairs on the current device
 * (wan_attn_pair_resident_clusters) are fullest once a split count's fill
 * is discounted by 6 %, the measured cost of the partials and the
 * combining pass.  Returns a negative wan_status on failure.              */
int wan_block_causal_attn_pair_splits(int B, int Lq, int Lk, int heads,
                                      int chunk_tokens, int q_offset);

/* How many CTA pairs of the pair kernels can be resident at once on the
 * current device (clusters of two CTAs must share a GPC, so an SM left over
 * in a GPC with an odd number of SMs runs none).  A diagnostic; returns a
 * negative wan_status on failure.                                          */
int wan_attn_pair_resident_clusters(void);

/* ---------------------------------------- block prologue and epilogue --
 * Wan2.2 source reading, ch. 4, section "Full forward of one block": the
 * self-attention input is norm1(x) * (1 + e[1]) + e[0] and the block output
 * x + y * e[2] (fp32 autocast); section "3D RoPE": q and k each pass an
 * RMSNorm (QK-Norm) after their linear layers, before the rotation.
 *
 * wan_adaln_modulate: out[b,l,:] = LN(x[b,l,:]) * (1 + scale[b,:])
 *   + shift[b,:], LN over D without affine weights, variance eps.  x fp32
 *   [B, L, D]; shift, scale fp32 [B, D]; out bf16 [B, L, D].  D % 4 == 0,
 *   D <= 8192, all pointers 16-byte aligned.
 * wan_qk_norm_rope: in place on q and k ([B, L, heads, 128] bf16, either may
 *   be NULL): t <- rope3d(t / sqrt(mean_{heads*128}(t^2) + eps) * w), the
 *   mean over all heads of a token, w fp32 [heads * 128] (wq for q, wk for
 *   k), then the 3D RoPE of grid g with the wan_rope3d_table layout.
 * wan_gated_residual: x[b,l,:] += y[b,l,:] * gate[b,:]; x fp32 [B, L, D],
 *   y bf16 [B, L, D] (8-byte aligned), gate fp32 [B, D].  D % 4 == 0.       */
int wan_adaln_modulate(const float* x, const float* shift, const float* scale,
                       void* out, int B, int L, int D, float eps, void* s);
int wan_qk_norm_rope(void* q, void* k, const float* wq, const float* wk,
                     int B, wan_grid_t g, int heads, int head_dim,
                     const void* d_table, float eps, void* s);
int wan_gated_residual(float* x, const void* y, const float* gate, int B,
                       int L, int D, void* s);

/* ------------------------------------------------------------- sampler --
 * Wan2.2 source reading, ch. 5, section "shift": the points are laid
 * uniformly and mapped by sigma = shift*s / (1 + (shift-1)*s); ch. 1
 * "One ruler, two scales": t = 1000 * sigma.
 * wan_fm_sigmas: host, fp64.  Writes sigma_0 .. sigma_N (n_steps + 1
 *   values) to sigmas_out with s_i = s_max * (1 - i/n_steps), i < n_steps,
 *   and sigma_N = 0.  n_steps >= 1, shift > 0, 0 < s_max <= 1.
 *
 * Wan2.2 source reading, ch. 5 "UniPC" (Euler: velocity held constant over
 * the step) and "CFG" (uncond + w * (cond - uncond)):
 * wan_fm_step: x[i] += (sigma_next - sigma) * v[i], with
 *   v = v_cond                                   if v_uncond == NULL,
 *   v = v_uncond + guide * (v_cond - v_uncond)   otherwise,
 *   all fp32 on the device, n elements, in place on x.  dt = sigma_next -
 *   sigma is formed in fp64 on the host and rounded once to fp32.  x, v_cond
 *   and v_uncond must be 16-byte aligned; x may not alias the velocities.  */
int wan_fm_sigmas(int n_steps, double shift, double s_max,
                  double* sigmas_out);
int wan_fm_step(float* x, const float* v_cond, const float* v_uncond,
                float guide, int64_t n, double sigma, double sigma_next,
                void* s);

/* -------------------------------------------------------------- UniPC ---
 * Wan2.2 source reading, ch. 5 "UniPC": the default sampler is a multistep
 * predictor-corrector of order 2; the predictor extrapolates the trend of
 * the last two model outputs, the corrector redoes the step just taken with
 * the new output (no extra forward).  Ch. 1: x = (1 - sigma) x0 + sigma
 * noise, clean estimate m = x - sigma v.  The pages give no coefficients:
 * they follow the published UniPC order conditions (data prediction,
 * lambda = log((1 - sigma) / sigma), coefficients solved exactly); the step
 * to sigma = 0 is first order and an earlier stop at sigma = 1 is dropped.
 *
 * wan_unipc_coeffs: host, fp64.  Folded coefficients of stop i (0 <= i <
 * n_steps) of the schedule sigmas[0 .. n_steps] (strictly decreasing, in
 * [0, 1], sigmas[n_steps] >= 0):
 *   m_i   = x~_i - sigma * v
 *   x^c_i = cx x^c_(i-1) + cm1 m_(i-1) + cm2 m_(i-2) + cm m_i  (corr_order
 *           1 or 2: differences used, the new point included; corr_order 0
 *           at i == 0, where x^c_0 = x~_0)
 *   x~_(i+1) = px x^c_i + pm m_i + pm1 m_(i-1)  (pred_order 1 or 2).
 *   WAN_EINVAL for a bad schedule or index.
 *
 * wan_unipc_step: device, fp32, n elements, one fused pass:
 *   v = v_cond, or v_uncond + guide * (v_cond - v_uncond) if v_uncond;
 *   x      in: x~_i      out: x~_(i+1)
 *   x_corr in: x^c_(i-1) (not read at i == 0)   out: x^c_i
 *   m_prev1 = m_(i-1) (read if i >= 1), m_prev2 = m_(i-2) (read if
 *   corr_order == 2), m_out receives m_i and may alias m_prev2 (a caller
 *   keeps two buffers and swaps them); no other pointers may alias.  All
 *   16-byte aligned (WAN_EALIGN); coefficients rounded once to fp32.       */
typedef struct {
  double sigma;
  double cx, cm1, cm2, cm;
  double px, pm, pm1;
  int32_t pred_order;
  int32_t corr_order;
} wan_unipc_coef_t;

int wan_unipc_coeffs(const double* sigmas, int n_steps, int i,
                     wan_unipc_coef_t* out);
int wan_unipc_step(float* x, float* x_corr, const float* m_prev1,
                   const float* m_prev2, float* m_out, const float* v_cond,
                   const float* v_uncond, float guide, int64_t n,
                   const double* sigmas, int n_steps, int i, void* s);

/* ------------------------------------------------------------ Ulysses ---
 * Wan2.2 source reading, ch. 8 "Ulysses": the multi-GPU split trades each
 * rank's sequence shard of all heads for the whole sequence of its share of
 * the heads (one all-to-all that scatters one dimension and gathers
 * another), runs attention, and trades back.
 *
 * wan_transpose_blocks: device.  out[j][i][:] = in[i][j][:] for i < a,
 *   j < b, each row row_bytes long: the outer-dimension swap that makes a
 *   rank's outgoing chunks (and incoming shards) contiguous around the
 *   all-to-all.  row_bytes a multiple of 16, in / out 16-byte aligned
 *   (WAN_EALIGN) and not overlapping (WAN_EINVAL).  Empty sizes do nothing.
 *   The exchange itself is NCCL's all-to-all.                              */
int wan_transpose_blocks(const void* in, void* out, int64_t a, int64_t b,
                         int64_t row_bytes, void* s);

/* ---------------------------------------------------- wait self-test ---
 * wan_wait_selftest: launches one warp on stream s that waits, with the
 * library's bounded mbarrier wait, on a barrier needing one arrival and
 * given `arrive` (0 or 1) of them.  With 0 the wait runs out after its 2 s
 * limit, WAN_ETIMEOUT is recorded in the device status word
 * (wan_device_status) and the kernel returns, leaving the context usable;
 * with 1 it completes at once.  It lets a test check the timeout path
 * without a fault or a hang.  The pages have no counterpart: this is a
 * check of the library's own failure handling.  WAN_EINVAL for other
 * values of arrive.                                                        */
int wan_wait_selftest(int arrive, void* s);

/* ------------------------------------------------------------- status ---
 * Reads (and, if clear != 0, resets) the device status word of the current
 * device: 0 or WAN_ETIMEOUT.  Synchronous (waits for the device).          */
int wan_device_status(int clear);

#ifdef __cplusplus
}
#endif

#endif /* WAN_H_ */
