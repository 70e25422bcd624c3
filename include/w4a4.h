/*
 * w4a4.h -- C ABI of the B200 (sm_100a) W4A4 NVFP4 linear layer.
 *
 * The operation is the dual-branch SVDQuant linear of a diffusion transformer
 * ("SVDQuant Guide: 4-Bit DiT Acceleration & Outlier Absorption", pillar 1
 * "Mathematical Outlier Factorization" and pillar 2 "SmoothQuant
 * Pre-Conditioning for DiTs"; section "Step 2: The SVDQuant Dual-Branch Linear
 * Layer"), written token-major:
 *
 *     Y = bf16( Q(X diag(s)^-1) Q(R)^T  +  (X L1) L2  +  bias )
 *
 *   X    [M, K]  bf16 activation, M tokens, K input channels
 *   s    [K]     smoothing factors (the caller passes inv_s = 1/s in fp32)
 *   R    [N, K]  residual of the smoothed weight after its rank-r part
 *   L1   [K, r]  low-rank down-projection, 1/s folded in (passed as L1t = L1^T [r, K])
 *   L2   [r, N]  low-rank up-projection (passed as L2t = L2^T [N, r])
 *   Q()  NVFP4 quantisation: E2M1 element codes {0,+-0.5,+-1,+-1.5,+-2,+-3,+-4,+-6},
 *        one unsigned E4M3 scale per 16 consecutive K elements, one fp32 scale
 *        per tensor.  NVFP4 is the format the pages name for FLUX on Blackwell
 *        ("NVIDIA Technical Blog Details FLUX 3 Image Klein Blackwell Inference
 *        Optimization Methods ...", first optimisation layer); its exact
 *        arithmetic is fixed below.
 *
 * Quantisation arithmetic (every step one correctly rounded fp32 operation):
 *   x~ = x * inv_s[k];  A = max |x~| over the tensor;
 *   t = A / 2688 (2688 = 6 * 448), t = 1 if that is not a normal fp32 number;
 *   per 16-block: b = max |x~|, scale byte e = E4M3_rn_satfinite((b * (1/t)) / 6);
 *   code = E2M1_rn_satfinite(x~ * (1 / (dec(e) * t))), all +0 if dec(e) == 0.
 *   Two codes per byte, the even K index in the low nibble.
 *
 * Memory layouts (all device memory, row-major unless stated):
 *   packed codes   [rows, K/2] uint8
 *   block scales   "SF atom" layout, nvfp4_sf_bytes(rows, K) bytes: rows are
 *                  grouped in blocks of 128 (the last block padded), K in groups
 *                  of 64 (4 scales).  Each (128-row block rb, 64-K group kg)
 *                  pair is a 512-byte atom at offset (rb * K/64 + kg) * 512;
 *                  inside it, the scale of row m and 16-block j (j = 0..3 in
 *                  the group) sits at byte (m % 32) * 16 + ((m / 32) % 4) * 4 + j.
 *                  This is the order in which the tensor cores read scales.
 *   U (low-rank)   [M, 2r] bf16: columns [0, r) hold hi = bf16(u'), columns
 *                  [r, 2r) hold lo = bf16(u' - hi), where u' = (X L1) / (t_x t_w)
 *                  in fp32.  hi + lo carries u' to about 16 significant bits.
 *
 * Conventions:
 *   - The caller owns every buffer.  No function allocates, frees or
 *     synchronises; all work is enqueued on `stream` (a cudaStream_t, NULL for
 *     the legacy default stream).  Scalars (t_x, t_w) stay in device memory.
 *   - Host-detectable problems return an error before anything is enqueued.
 *   - Pointers must be 16-byte aligned; ldx/ldr/ldy are in elements.
 *   - Constraints: K % 64 == 0, 64 <= K <= W4A4_MAX_K (one FP4 MMA K-step of
 *     four 16-element scale blocks; the bound is the widest row the
 *     tensor-amax pass covers with its fixed count of partial maxima);
 *     N % 8 == 0; r in {0, 16, 32}
 *     (rank 16 is the pages' choice for the low-rank branch, "SVDQuant
 *     Guide ...", "The Solution ..." and "Empirical Efficiency Benchmark");
 *     M >= 0, rows need not be a multiple of 128.  An empty problem (M == 0;
 *     N == 0 for nvfp4_pack_weight; rows == 0 for nvfp4_sf_to_rowmajor) with
 *     valid sizes returns W4A4_OK at once: pointers may then be NULL,
 *     nothing is checked further and nothing is enqueued.
 *   - A device-side pipeline wait that exceeds its bound (about two seconds,
 *     see w4a4_set_wait_bound) records W4A4_ERR_DEVICE_TIMEOUT in a sticky
 *     status word, drains its own copies and returns; read it with
 *     w4a4_device_status().
 *   - The current CUDA device must be compute capability 10.x (B200 / sm_100a);
 *     there is no fallback.
 */
#ifndef W4A4_H_
#define W4A4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  W4A4_OK = 0,
  W4A4_ERR_NULL = -1,           /* a required pointer is NULL */
  W4A4_ERR_SHAPE = -2,          /* unsupported size or rank */
  W4A4_ERR_ALIGN = -3,          /* pointer or leading dimension not 16-byte aligned */
  W4A4_ERR_ARCH = -4,           /* no CUDA device, or not compute capability 10.x */
  W4A4_ERR_WORKSPACE = -5,      /* workspace NULL or smaller than required */
  W4A4_ERR_CUDA = -6,           /* a CUDA call or kernel launch failed */
  W4A4_ERR_DEVICE_TIMEOUT = -7, /* sticky device status: a bounded wait gave up */
  W4A4_ERR_ARG = -8,            /* an enum argument is out of range */
  W4A4_ERR_SCRATCH_LIMIT = -9,  /* problem needs more than the built-in scratch (no-alloc entry) */
  W4A4_ERR_DEVICE_LAYOUT = -10  /* sticky device status: a kernel found its shared memory misaligned */
} w4a4_status;

/* Largest K (columns of an activation or weight) every entry point accepts. */
#define W4A4_MAX_K ((int64_t)1 << 20)

enum { W4A4_EPI_NONE = 0, W4A4_EPI_GELU_TANH = 1 };
enum { W4A4_SRC_BF16 = 0, W4A4_SRC_F32 = 1 };

/* Bytes of the SF-atom block-scale buffer for a [rows, K] tensor:
 * ceil(rows / 128) * 128 * K / 16.  Returns 0 for invalid sizes. */
size_t nvfp4_sf_bytes(int64_t rows, int64_t K);

/* Workspace bytes needed by nvfp4_quantize_act / nvfp4_pack_weight for an
 * [M, K] input with rank r (amax partial maxima, the grid-barrier words of the
 * single-pass quantiser, per-row-block counters and low-rank partial sums).
 * Returns 0 for invalid sizes.
 *
 * Workspace contract (every entry point that takes a workspace): zero the
 * whole workspace once before its first use (cudaMemset, torch.zeros).  The
 * synchronisation words in it stay valid from call to call (counters are
 * cleared by the call that used them; the single-pass grid barrier keeps a
 * launch generation that every call advances), so no clearing is needed
 * between calls, whatever their sizes: the layout below is the same for every
 * M, K and r, only the length of the last part grows with M.  After a call
 * reports a device error (w4a4_device_status), zero the workspace again: a
 * wait that gave up leaves its counters where they stood.  Calls that overlap
 * on the GPU must not share a workspace.
 *
 * Layout (byte offsets from the workspace base):
 *   0                        amax partial maxima of the two-pass path (fp32 x 1024)
 *   W4A4_WS_BARRIER_OFFSET   grid barrier: launch generation, arrival counters
 *                            and tensor-maximum words (160 u32, 128-byte lines)
 *   W4A4_WS_TICKETS_OFFSET   one u32 counter per 128-row block (row block b at
 *                            byte W4A4_WS_TICKETS_OFFSET + 4 b), zero at rest
 *   W4A4_WS_UPART_OFFSET     fp32 low-rank partial sums (r > 0 only)
 * With a low-rank branch (r > 0) M is at most W4A4_MAX_LOWRANK_ROWS, the
 * number of rows the counters cover. */
#define W4A4_WS_BARRIER_OFFSET ((size_t)4096)
#define W4A4_WS_TICKETS_OFFSET ((size_t)5120)
#define W4A4_MAX_LOWRANK_ROWS ((int64_t)1 << 22)
#define W4A4_WS_UPART_OFFSET (W4A4_WS_TICKETS_OFFSET + (size_t)4 * (size_t)(W4A4_MAX_LOWRANK_ROWS / 128))
size_t nvfp4_quant_workspace_bytes(int64_t M, int64_t K, int r);

/* Workspace bytes needed by w4a4_linear: the quantisation workspace plus the
 * quantised activation (codes, scales, t_x) and the low-rank U buffer. */
size_t w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/*
 * nvfp4_quantize_act -- online activation quantisation (smooth, tensor amax,
 * block scales, codes, packing) fused with the low-rank down-projection.
 * Activations are quantised afresh at every denoising step because their
 * outlier channels drift with the timestep ("SVDQuant Guide ...", section
 * "Why Standard Low-Bit Quantization Fails on DiTs", "Timestep-Dynamic
 * Activation Drift").
 *
 *   X      in   bf16 [M, ldx] row-major, the first K columns are used
 *   inv_s  in   fp32 [K] reciprocal smoothing factors, NULL = all ones
 *   L1t    in   bf16 [r, K] (NULL iff r == 0)
 *   t_w    in   fp32 device scalar, the weight's tensor scale (needed iff r > 0)
 *   Xq     out  uint8 [M, K/2] packed E2M1 codes
 *   Xsf    out  uint8 SF-atom layout, nvfp4_sf_bytes(M, K) bytes (pad rows get 0)
 *   t_x    out  fp32 device scalar, the activation's tensor scale
 *   U      out  bf16 [M, 2r] hi/lo low-rank activations (NULL iff r == 0)
 *   workspace   >= nvfp4_quant_workspace_bytes(M, K, r) bytes of device memory,
 *               zeroed before its first use (see nvfp4_quant_workspace_bytes);
 *               must not overlap the outputs
 * Launches one cooperative kernel (tensor amax, grid barrier, quantise and
 * down-projection) when every (128-row block, K slice) tile of X fits on the
 * device at once, otherwise two (tensor amax, then quantise + down-projection).
 */
int nvfp4_quantize_act(const void* X, int64_t M, int64_t K, int64_t ldx,
                       const float* inv_s, const void* L1t, int r, const float* t_w,
                       uint8_t* Xq, uint8_t* Xsf, float* t_x, void* U,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * nvfp4_quantize_act_with_amax -- nvfp4_quantize_act with the activation's
 * tensor amax A = max |fl(x * inv_s)| supplied by the caller (normally
 * written by w4a4_gemm_next_amax, the producer of X) instead of measured: the
 * quantiser then streams X once at any size.  The result is bit-identical to
 * nvfp4_quantize_act when *amax equals the measured amax.  Same arguments as
 * nvfp4_quantize_act plus
 *   amax  in  fp32 device scalar (4-byte aligned), A >= 0
 * W4A4_ERR_NULL if amax is NULL, W4A4_ERR_ALIGN if misaligned.  Launches one
 * quantise kernel.
 */
int nvfp4_quantize_act_with_amax(const void* X, int64_t M, int64_t K, int64_t ldx,
                                 const float* inv_s, const void* L1t, int r, const float* t_w,
                                 const float* amax, uint8_t* Xq, uint8_t* Xsf, float* t_x, void* U,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * nvfp4_pack_weight -- offline NVFP4 packing of the residual weight R [N, K]
 * (bf16 or fp32 source, row stride ldr elements) with the same quantiser
 * (no smoothing: the smoothing factors are already multiplied into R).  The
 * pages quantise the residual after removing the low-rank part ("SVDQuant
 * Guide ...", "Step 1: Low-Rank Outlier Decomposition in PyTorch").
 *   Wq out uint8 [N, K/2]; Wsf out nvfp4_sf_bytes(N, K) bytes; t_w out fp32 scalar.
 */
int nvfp4_pack_weight(const void* R, int src_dtype, int64_t N, int64_t K, int64_t ldr,
                      uint8_t* Wq, uint8_t* Wsf, float* t_w,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * w4a4_gemm -- block-scaled FP4 GEMM on the tcgen05 tensor cores fused with
 * the low-rank up-projection, bias and the bf16 cast (the fused 4-bit +
 * low-rank kernel of "SVDQuant Guide ...", pillar 3 "The Nunchaku Fused Kernel
 * Engine", re-designed for sm_100a):
 *   Y[m,n] = bf16( t_x t_w ( sum_k dec(Xq) dec(Xsf) dec(Wq) dec(Wsf)
 *                            + sum_j U[m,j] L2t[n,j] ) + bias[n] )
 * with U the hi/lo pair written by nvfp4_quantize_act (so the low-rank term is
 * (X L1) L2 after the t_x t_w factor).  epilogue = W4A4_EPI_GELU_TANH applies
 * 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))) before the bf16 cast.
 *   Xq/Xsf/t_x/U  in  as written by nvfp4_quantize_act (U NULL iff r == 0)
 *   Wq/Wsf/t_w    in  as written by nvfp4_pack_weight
 *   L2t  in  bf16 [N, r] (NULL iff r == 0);  bias in bf16 [N] or NULL
 *   Y    out bf16 [M, ldy], ldy >= N, ldy % 8 == 0
 * The kernel is launched with programmatic stream serialisation: its set-up
 * (barriers, TMEM allocation) overlaps the end of the previous kernel in the
 * stream, and it touches no memory before that kernel has completed.
 */
int w4a4_gemm(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U,
              int64_t M, int64_t N, int64_t K,
              const uint8_t* Wq, const uint8_t* Wsf, const float* t_w,
              const void* L2t, int r, const void* bias, int epilogue,
              void* Y, int64_t ldy, void* stream);

/*
 * w4a4_gemm_next_amax -- w4a4_gemm that also measures the tensor amax the
 * next layer's activation quantiser needs when Y is that activation (the
 * fused producer epilogue of "NVIDIA Technical Blog Details FLUX 3 Image Klein
 * Blackwell Inference Optimization Methods": NVFP4 with fused GEMM
 * epilogues): over the stored bf16 outputs (after bias and GELU),
 *   *next_amax = max(*next_amax, max_{m,n} |fl(Y[m,n] * next_inv_s[n])|)
 * as an atomic maximum on the value's bit pattern.  Same arguments as
 * w4a4_gemm plus
 *   next_inv_s  in     fp32 [N] reciprocal smoothing factors of the next
 *                      layer (> 0), 16-byte aligned, or NULL for all ones
 *   next_amax   in/out fp32 device scalar, 4-byte aligned; must hold a
 *                      non-negative value on entry (normally 0)
 * W4A4_ERR_NULL if next_amax is NULL, W4A4_ERR_ALIGN if misaligned.
 */
int w4a4_gemm_next_amax(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U,
                        int64_t M, int64_t N, int64_t K, const uint8_t* Wq, const uint8_t* Wsf,
                        const float* t_w, const void* L2t, int r, const void* bias, int epilogue,
                        void* Y, int64_t ldy, const float* next_inv_s, float* next_amax,
                        void* stream);

/*
 * w4a4_gemm_swiglu -- w4a4_gemm for a fused projection whose last output
 * features are SwiGLU gate/up pairs: the kernel applies the SwiGLU epilogue
 * that the NVIDIA blog page on FLUX on Blackwell fuses into its NVFP4 GEMM
 * ("NVIDIA Technical Blog Details FLUX 3 Image Klein Blackwell Inference
 * Optimization Methods", the NVFP4 / fused-GEMM paragraph), so the gate and
 * up features never reach memory.  With y[m,n] = t_x t_w acc[m,n] + bias[n]
 * in fp32 (acc as in w4a4_gemm, over the packed weight rows n):
 *   rows n < n_plain:   Y[m,n] = bf16(y[m,n])
 *   rows n >= n_plain:  grouped in blocks of 32, block b = 16 gate rows
 *                       n_plain + 32b + i and then the 16 up rows
 *                       n_plain + 32b + 16 + i (i = 0..15) of output
 *                       features j = 16b + i:
 *                       H[m,j] = bf16(silu(y[m, gate row]) * y[m, up row]),
 *                       silu(v) = v / (1 + exp(-v))
 * (the Python package's prep.swiglu_row_order gives the row order for a weight laid
 * out [plain | gate | up]).  Same arguments as w4a4_gemm, without epilogue,
 * plus
 *   n_plain     plain output features, a multiple of 256, 0 <= n_plain < N;
 *               (N - n_plain) a multiple of 32
 *   Y, ldy      bf16 [M, ldy], ldy >= n_plain (Y may be NULL iff n_plain == 0)
 *   H, ldh      bf16 [M, ldh], ldh >= (N - n_plain) / 2, ldh % 8 == 0
 *   next_inv_s, next_amax  as in w4a4_gemm_next_amax, over H only (the next
 *               layer's input; next_inv_s indexed by H's column), or
 *               next_amax NULL for none
 * Launches one CTA-pair GEMM kernel.
 */
int w4a4_gemm_swiglu(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U,
                     int64_t M, int64_t N, int64_t K, const uint8_t* Wq, const uint8_t* Wsf,
                     const float* t_w, const void* L2t, int r, const void* bias, int64_t n_plain,
                     void* Y, int64_t ldy, void* H, int64_t ldh, const float* next_inv_s,
                     float* next_amax, void* stream);

/*
 * w4a4_gemm_rope -- w4a4_gemm_swiglu whose epilogue also applies the rotary
 * position embedding to the leading query/key features, the third epilogue
 * the NVIDIA blog page on FLUX on Blackwell names for its fused NVFP4 GEMM
 * ("NVIDIA Technical Blog Details FLUX 3 Image Klein Blackwell Inference
 * Optimization Methods", the NVFP4 / fused-GEMM paragraph: SwiGLU, QKV
 * projection and RoPE epilogues).  The page gives no formula; this is the
 * rotation of adjacent feature pairs by per-token, per-pair angles given as a
 * table (any 1-D or multi-axis angle schedule reduces to one).  Rows n <
 * n_rope form n_rope / d_head heads of d_head features; in every head,
 * features 2i and 2i+1 (i = 0 .. d_head/2 - 1) are the pair i.  With y as in
 * w4a4_gemm_swiglu (fp32, t_x t_w acc + bias) and, for token m and pair i,
 * c = rope[m * ld_rope + 2i], s = rope[m * ld_rope + 2i + 1]
 * (cos and sin of its angle):
 *   Y[m, head + 2i]     = bf16(y[m, head + 2i] c - y[m, head + 2i + 1] s)
 *   Y[m, head + 2i + 1] = bf16(y[m, head + 2i] s + y[m, head + 2i + 1] c)
 * one rounding of the rotated fp32 value (the values are not rounded to bf16
 * before the rotation).  Rows n_rope <= n < n_plain are plain outputs, rows
 * n >= n_plain SwiGLU pairs, exactly as in w4a4_gemm_swiglu.  Same arguments
 * as w4a4_gemm_swiglu plus
 *   n_rope      rotated features, 0 < n_rope <= n_plain, a multiple of d_head
 *   d_head      features per head, a multiple of 32
 *   rope        in fp32 [M, ld_rope]: per token the d_head/2 (cos, sin) pairs
 *               of its head features, the same for every head; 16-byte aligned
 *   ld_rope     row stride of rope in floats, >= d_head, a multiple of 4
 * and n_plain may equal N (no SwiGLU features; H NULL, next_amax over Y).
 * With n_plain < N it must be a multiple of 256, as in w4a4_gemm_swiglu.
 * W4A4_ERR_SHAPE for sizes outside these ranges, W4A4_ERR_NULL for a NULL
 * rope, W4A4_ERR_ALIGN for a misaligned one.  Launches one CTA-pair GEMM
 * kernel.
 */
int w4a4_gemm_rope(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U,
                   int64_t M, int64_t N, int64_t K, const uint8_t* Wq, const uint8_t* Wsf,
                   const float* t_w, const void* L2t, int r, const void* bias,
                   int64_t n_rope, int64_t d_head, const float* rope, int64_t ld_rope,
                   int64_t n_plain, void* Y, int64_t ldy, void* H, int64_t ldh,
                   const float* next_inv_s, float* next_amax, void* stream);

/*
 * w4a4_gemm_quantize_next -- w4a4_gemm (epilogue NONE or GELU_TANH) or
 * w4a4_gemm_swiglu (n_plain < N) whose epilogue also quantises its final
 * outputs for the next layer, so that layer's activation quantiser need not
 * read them: the fusion the SVDQuant guide's engine section motivates ("SVDQuant
 * Guide: 4-Bit DiT Acceleration & Outlier Absorption", "3. The Nunchaku Fused
 * Kernel Engine": no second kernel streaming the same tensor), under a tensor
 * scale the caller gives (a static calibration, "1. Timestep-Aware Outlier
 * Calibration", or the previous step's), which is what makes it possible in
 * one pass: the scale no longer comes from this step's amax.
 *   The final outputs F are Y (n_plain == N; after bias and the epilogue) or
 *   H (the SwiGLU outputs).  Column c of F is column next_col + c of the next
 *   layer's [M, next_K] activation; for every row m and 16-block of F, with
 *   x~ = fl(bf16(F[m,c]) * next_inv_s[c]) and t = *next_t, the kernel writes
 *   the scale byte E4M3_rn_satfinite((b * (1/t)) / 6) and the codes
 *   E2M1_rn_satfinite(x~ * (1 / (dec(e) t))) (+0 for a zero scale) of
 *   nvfp4_quantize_act -- bit for bit what nvfp4_quantize_act would write for
 *   these columns of the bf16 outputs if its tensor scale were t.
 *   next_inv_s  in   fp32 [n_out] (n_out = N, or (N - n_plain) / 2), or NULL for ones
 *   next_t      in   fp32 device scalar, the next layer's tensor scale (> 0,
 *                    a normal number); pass it as that layer's t_x
 *   next_q      out  uint8 codes [M, next_ldq bytes], next_ldq >= next_K / 2,
 *                    next_ldq % 16 == 0; bytes [next_col / 2, (next_col + n_out) / 2)
 *                    of each row are written
 *   next_sf     out  SF atoms of the [M, next_K] activation (nvfp4_sf_bytes(M,
 *                    next_K) bytes); the scale bytes of those columns for rows
 *                    < M are written (pad rows are left as they are)
 *   next_K, next_col  next_K % 64 == 0, next_K <= W4A4_MAX_K, next_col % 64 == 0,
 *                    next_col + n_out <= next_K
 *   next_amax   as in w4a4_gemm_next_amax (over F), or NULL
 *   Y / H       as in w4a4_gemm / w4a4_gemm_swiglu; may be NULL to skip
 *               storing the bf16 values (Y must be given when n_plain is
 *               between 0 and N: those outputs are not quantised)
 * The next layer's low-rank input U = F L1 still needs the bf16 F (the
 * quantiser with the amax given computes it); a next layer without a
 * low-rank branch needs only next_q, next_sf and next_t.  n_out % 32 == 0.
 * Launches one CTA-pair GEMM kernel.
 */
int w4a4_gemm_quantize_next(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U,
                            int64_t M, int64_t N, int64_t K, const uint8_t* Wq, const uint8_t* Wsf,
                            const float* t_w, const void* L2t, int r, const void* bias, int epilogue,
                            int64_t n_plain, void* Y, int64_t ldy, void* H, int64_t ldh,
                            const float* next_inv_s, const float* next_t, uint8_t* next_q,
                            int64_t next_ldq, uint8_t* next_sf, int64_t next_K, int64_t next_col,
                            float* next_amax, void* stream);

/*
 * FP8 attention.  The NVIDIA blog page on FLUX on Blackwell quantises the
 * attention that consumes the fused projection's queries, keys and values to
 * FP8 ("NVIDIA Technical Blog Details FLUX 3 Image Klein Blackwell Inference
 * Optimization Methods", the paragraph on quantised and sparse attention:
 * VC-Attention FP8) and states no arithmetic; the reading implemented here is
 * per-tensor E4M3 quantisation of Q, K and V and the exact softmax attention
 * of the dequantised tensors, evaluated on the FP8 tensor cores.  The page's
 * "repair budget" is not defined there and is not implemented.
 *
 * fp8_quantize -- one bf16 tensor X [rows, cols] (row stride ldx elements) to
 * E4M3 codes with one fp32 scale s = amax / 448 (1 when that is not a normal
 * number), code = E4M3_rn_satfinite(fl(x * fl(1/s))), written row-major
 * (out[r * ldo + c], transpose = 0) or transposed (out[c * ldo + r],
 * transpose = 1: the value layout attention_fp8 reads).  Two kernels: the
 * tensor amax into the workspace, then the codes.
 *   cols % 8 == 0, cols <= 2^21, ldx >= cols, ldx % 8 == 0; transpose: rows % 16 == 0,
 *   ldo >= rows, ldo % 16 == 0; else ldo >= cols, ldo % 8 == 0
 *   scale     out fp32 device scalar (4-byte aligned)
 *   workspace >= fp8_quant_workspace_bytes(rows, cols) bytes of device memory
 *             (no zeroing needed)
 * W4A4_ERR_SHAPE / _NULL / _ALIGN / _WORKSPACE on bad arguments; rows == 0
 * enqueues nothing.
 */
size_t fp8_quant_workspace_bytes(int64_t rows, int64_t cols);
int fp8_quantize(const void* X, int64_t rows, int64_t cols, int64_t ldx, int transpose,
                 uint8_t* out, int64_t ldo, float* scale, void* workspace, size_t workspace_bytes,
                 void* stream);

/*
 * attention_fp8 -- O = softmax(c Q K^T) V per head and sequence, on E4M3
 * operands: batch sequences of S tokens (S % 128 == 0, batch * S <= 2^30),
 * heads of 128 features.
 *   Q8, K8  in  E4M3 [batch * S, ldq / ldk bytes], token-major, head h in
 *               columns h*128 .. h*128+127 (ld >= heads*128, ld % 16 == 0)
 *   Vt8     in  E4M3 [heads * 128, ldvt bytes]: V transposed, row h*128 + d,
 *               column b*S + j (ldvt >= batch*S, ldvt % 16 == 0), as written
 *               by fp8_quantize with transpose = 1
 *   s_q, s_k, s_v  in fp32 device scalars: the tensors' dequantisation scales
 *   softmax_scale  c (normally 1/sqrt(128)), finite and > 0
 *   O       out bf16 [batch * S, ldo], head h in columns h*128 .. (ldo % 8 == 0)
 * The kernel computes S = Q K^T on the tensor cores in fp32, an online
 * softmax in fp32 with the probabilities rounded to E4M3 (within 2^-17 to
 * 2^8.5 of the row's running maximum) for the second product O += P V, and
 * writes bf16(O s_v / l), l the sum of the probabilities before their
 * rounding (unbiased, so it differs from the sum of the rounded ones far
 * less than the rounding changes each product).  One CTA
 * per (128 queries, head, sequence), two per SM; programmatic stream
 * serialisation as for the GEMMs.
 */
int attention_fp8(const uint8_t* Q8, const uint8_t* K8, const uint8_t* Vt8, int64_t batch, int64_t S,
                  int64_t heads, int64_t ldq, int64_t ldk, int64_t ldvt, const float* s_q,
                  const float* s_k, const float* s_v, float softmax_scale, void* O, int64_t ldo,
                  void* stream);

/*
 * w4a4_fp4_mma_rate -- a measurement, not part of the layer: the rate of the
 * block-scaled FP4 tensor-core instruction the GEMM is built on
 * (tcgen05.mma kind::mxf4nvf4.block_scale.block16), issued back to back with
 * resident operands (pseudo-random codes, scale bytes 0x30..0x3F) on every
 * SM.  It gives the measured FP4 peak beside the nominal one; the pages quote
 * the FP4 tensor-core speedup only as a ratio ("Four Bits ...": 4x over FP16).
 *   iters   MMAs per issuing thread, 1 .. 2^20
 *   pair    1: 256 x 256 x 64 MMAs on CTA pairs (cta_group::2, one issuer per
 *           two SMs); 0: 128 x 256 x 64 MMAs, one CTA and issuer per SM
 *   cycles  out: device array of at least (number of SMs) entries; entry i is
 *           the SM clock cycles issuer i took for its MMAs, from its first
 *           issue to the completion of its last (0 if its wait gave up)
 * One kernel on `stream`; time it with events to get the rate in FLOP/s
 * (2 * 256 * 256 * 64 or 2 * 128 * 256 * 64 FLOPs per MMA).
 */
int w4a4_fp4_mma_rate(int iters, int pair, unsigned long long* cycles, void* stream);

/*
 * w4a4_linear -- the whole hot path: nvfp4_quantize_act on X (row stride K)
 * into the workspace, then w4a4_gemm into Y (row stride N).
 *   workspace >= w4a4_workspace_bytes(M, N, K, r) bytes of device memory.
 */
int w4a4_linear(const void* X, int64_t M, int64_t N, int64_t K,
                const uint8_t* Wq, const uint8_t* Wsf, const float* t_w,
                const float* inv_s, const void* L1t, const void* L2t, int r,
                const void* bias, int epilogue, void* Y,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * nvfp4_quantize_act_noalloc -- nvfp4_quantize_act for callers that cannot
 * allocate device memory.  The paper has no counterpart to this entry point;
 * it exists for hosts that hand a layer only its inputs and outputs: for
 * example an inference-engine plugin interface with no workspace slot, or a
 * serving runtime that plans every device buffer ahead of time and forbids
 * allocation while requests are in flight (cudaMalloc can synchronise the
 * device and fragment the planned memory).
 *
 * Arguments, layouts and results are those of nvfp4_quantize_act, without
 * the workspace: the scratch this computation needs (per-CTA amax partial
 * maxima, per-row-block counters and fp32 low-rank partial sums) lives in a
 * file-scope device array of W4A4_NOALLOC_SCRATCH_BYTES (16 MiB) built into
 * the library; every GPU that loads the library holds that array until the
 * process exits.  The entry point allocates nothing (no cudaMalloc, cudaFree
 * or allocating library call).
 *
 * - Sizes whose scratch need, nvfp4_quant_workspace_bytes(M, K, r), exceeds
 *   W4A4_NOALLOC_SCRATCH_BYTES are rejected with W4A4_ERR_SCRATCH_LIMIT
 *   before anything is enqueued (with r = 32 this admits M up to about
 *   65,000 rows at any K; r = 0 needs only the fixed header).
 * - Every call looks up the device address of the array on the current
 *   device (cudaGetSymbolAddress, with that device current); the first call
 *   for that address zeroes the array on the call's stream, so make the first
 *   call on a device before any stream capture.
 * - All calls share the one array, which keeps the last call's contents.  The
 *   kernels rewrite every scratch value they read and leave the counters zero
 *   when they end, so no clearing is needed between calls of any sizes (the
 *   scratch layout does not depend on them; see nvfp4_quant_workspace_bytes),
 *   but calls that overlap on the GPU (for example on two streams without
 *   ordering between them) race on the array and give wrong results.
 * - After a call reports a device error, w4a4_device_status(&st, 1) makes the
 *   next call on that device zero the array again before it runs.
 */
#define W4A4_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int nvfp4_quantize_act_noalloc(const void* X, int64_t M, int64_t K, int64_t ldx,
                               const float* inv_s, const void* L1t, int r, const float* t_w,
                               uint8_t* Xq, uint8_t* Xsf, float* t_x, void* U, void* stream);

/* Copies the sticky device status word of the current device into *status
 * (W4A4_OK, W4A4_ERR_DEVICE_TIMEOUT or W4A4_ERR_DEVICE_LAYOUT) and clears it
 * if reset != 0; a reset also makes the next nvfp4_quantize_act_noalloc call
 * on this device zero its built-in scratch first (caller-owned workspaces the
 * caller zeroes itself).  This call synchronises the device.  Returns W4A4_OK
 * or W4A4_ERR_CUDA. */
int w4a4_device_status(int* status, int reset);

/*
 * w4a4_last_error -- the sticky device status word of the current device
 * (W4A4_OK, W4A4_ERR_DEVICE_TIMEOUT or W4A4_ERR_DEVICE_LAYOUT), read without
 * synchronising the device: call it after synchronising the streams whose
 * work it should cover.  Does not clear the word (w4a4_device_status with
 * reset does).  W4A4_ERR_CUDA if the read itself fails.
 */
int w4a4_last_error(void);

/* Sets how long a device-side wait (pipeline barrier, grid barrier, counter)
 * spins before it gives up, records W4A4_ERR_DEVICE_TIMEOUT in the sticky
 * status word, drains its own copies and returns: ``cycles`` SM clock cycles
 * (at least 1e6), or the default 4e9 (about two seconds at 1.9 GHz) when
 * cycles <= 0.  Applies to kernels launched on the current device after the
 * call; synchronises the device.  A short bound lets a caller detect a stuck
 * pipeline quickly; it must stay well above the longest legitimate wait (a
 * full-size TMA stage lands within microseconds).  W4A4_ERR_ARG for
 * 0 < cycles < 1e6. */
int w4a4_set_wait_bound(int64_t cycles);

/*
 * nvfp4_sf_to_rowmajor -- a layout helper (for checking and debugging): the
 * block-scale bytes of an SF-atom buffer (nvfp4_sf_bytes(rows, K) bytes, as
 * written by nvfp4_quantize_act / nvfp4_pack_weight) rearranged row-major,
 * sf_rowmajor[m * (K/16) + k/16] = the E4M3 scale of row m, K-block k/16, for
 * the first ``rows`` rows (the atom layout's pad rows are dropped).  Device
 * pointers, stream-ordered, one kernel.  W4A4_ERR_SHAPE for invalid sizes,
 * W4A4_ERR_NULL / W4A4_ERR_ALIGN for bad pointers (16-byte alignment).
 */
int nvfp4_sf_to_rowmajor(const uint8_t* sf_atoms, int64_t rows, int64_t K, uint8_t* sf_rowmajor, void* stream);

/* Static description of a status code; never NULL. */
const char* w4a4_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* W4A4_H_ */
