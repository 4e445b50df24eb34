/*
 * dit3d.h -- C ABI of libdit3d: the hot path of a video Diffusion Transformer
 * block on NVIDIA B200 (sm_100a).
 *
 *   u   = LayerNorm(x) * (s0 + gamma_g) + beta_g            dit_adaln_modulate
 *   q,k = R3D(t, h, w) q,  R3D(t, h, w) k                     dit_rope3d_qk
 *   o   = softmax(q_rot k_rot^T / sqrt(d_head)) v             dit_attn_fwd
 *   out = x + alpha_g * y                                     dit_gated_residual
 *   x  += dt_frame * u   (sampler step, not in the block)       dit_flow_euler_step
 *   out = res + alpha_g * act(x w^T + b)  (projections, MLP)     dit_linear
 *   o   = attention on E4M3 q, k (and v, P)                     dit_attn_fwd_qk8 / _fp8
 *   q8  = e4m3(x * inv_scale)                                   dit_quantize_e4m3
 *   q8,k8 = e4m3(R3D q * inv_q), e4m3(R3D k * inv_k)               dit_rope3d_qk_e4m3
 *
 * Formulas: "DiT, Flow Matching e 3D Attention: A Engenharia de Video com IA",
 * sections "A ruptura da U-Net" (adaLN-Zero) and "3D-RoPE e atencao
 * espaco-temporal" (band split of the head dimension, rotated q/k, attention);
 * "Por que e absurdamente dificil gerar um filme inteiro usando IA", section
 * "Matematica por tras" (softmax(QK^T/sqrt(d))V).
 *
 * Conventions shared by every call
 *  - Tensors are dense, row-major, token-major bf16 in device memory, with no
 *    strides: activations [rows, D]; q/k/v/o [rows, H, d] (= [rows, D], D = H*d).
 *    The FP8 calls take the same layouts with one E4M3 code (byte) per element.
 *  - Every tensor pointer must be 16-byte aligned (128-bit loads and TMA); the
 *    exceptions are stated at their calls (fp32 lse and dt: 4 bytes; the codes
 *    written by dit_quantize_e4m3: 8 bytes).
 *  - The caller owns every buffer. Calls allocate nothing per call; the RoPE
 *    cos/sin tables (angles in fp64, stored fp32, written by a kernel) are cached in
 *    device memory per (device, descriptor, extent) on first use and freed by
 *    dit_shutdown(). The first call for a given RoPE descriptor allocates and waits for
 *    its table: make it outside CUDA-graph capture. Likewise the first attention call
 *    on a device whose dense batch gets its last wave split (see dit_attn_fwd) asks
 *    the occupancy calculator how many clusters fit, once per cluster size; make a
 *    call of the same shape before capturing one.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Calls only enqueue
 *    work: they return before the GPU has run it. Validation reads host data only.
 *  - Return value: DIT_OK or a dit_status code; nothing is printed, thrown or
 *    exited. Nothing is launched when validation fails.
 *  - Sequence layout (RoPE and attention). Dense: cu_seqlens_* = NULL and the
 *    rows form n_seq equal sequences of rows / n_seq tokens. Packed (varlen):
 *    cu_seqlens_host and cu_seqlens_dev both hold the same n_seq + 1 int32
 *    exclusive prefix sums (cu[0] = 0, non-decreasing, cu[n_seq] = rows).
 *  - Token order inside a sequence: row-major over the patch grid, t slowest,
 *    w fastest: token j has w = j % grid_w, h = (j / grid_w) % grid_h,
 *    t = j / (grid_h * grid_w). Positions restart at 0 for every sequence.
 */
#ifndef DIT3D_H_
#define DIT3D_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum dit_status {
  DIT_OK = 0,
  DIT_ERR_NULL = 1,     /* a required pointer is NULL                                  */
  DIT_ERR_SHAPE = 2,    /* unsupported or inconsistent sizes (see each call)            */
  DIT_ERR_ALIGN = 3,    /* a device pointer is not 16-byte aligned                      */
  DIT_ERR_SEQLENS = 4,  /* cu_seqlens not 0-based, decreasing, or not ending at rows    */
  DIT_ERR_DEVICE = 5,   /* current device is not sm_100 (B200 class)                     */
  DIT_ERR_LAUNCH = 6,   /* a CUDA call or kernel launch failed                          */
  DIT_ERR_TIMEOUT = 7,  /* a kernel's bounded wait expired (reported by dit_check_device) */
  DIT_ERR_ALLOC = 8,    /* the RoPE table cache could not allocate device memory        */
  DIT_ERR_SCRATCH = 9   /* dit_attn_fwd_noalloc: the RoPE table exceeds its fixed array  */
};

/* 3D-RoPE descriptor (DiT page, section "3D-RoPE e atencao espaco-temporal"):
 * the head dimension is cut into contiguous bands [t | h | w] of widths d_t, d_h,
 * d_w (each even, d_t + d_h + d_w = head_dim). In band a, the pair
 * (v[o_a+2i], v[o_a+2i+1]) turns by pos_a * base^(-2i/d_a) with the rotation
 * [[cos, -sin], [sin, cos]]; pos_a is the token's patch coordinate plus the
 * offset (t0, h0, w0). The frequency law, base and pair layout are this
 * library's reading: the pages give only the band split. */
typedef struct dit_rope3d_desc {
  int32_t grid_h, grid_w; /* patch-grid height H_lat/p_h and width W_lat/p_w (>= 1)      */
  int32_t d_t, d_h, d_w;  /* band widths, even, summing to head_dim                        */
  float base;             /* frequency base, > 1 (10000 in the workloads)                  */
  int32_t t0, h0, w0;     /* position offsets added to every token (>= 0)                   */
} dit_rope3d_desc;

/* adaLN modulation before attention or MLP (DiT page, "A ruptura da U-Net"):
 *   out[r, c] = (x[r,c] - mean_r) / sqrt(var_r + eps) * (scale_offset + gamma[g, c]) + beta[g, c]
 * with g = r / rows_per_group, LayerNorm over the D features of row r, biased
 * variance, fp32 statistics, no learned affine. scale_offset = 1 gives
 * LN(x)(1+gamma)+beta; 0 gives the page's gamma*LN(x)+beta.
 *   x, out      : [rows, D] bf16 (out may alias x)
 *   gamma, beta : [rows / rows_per_group, D] bf16
 * Errors: DIT_ERR_SHAPE unless rows >= 0, D > 0, D % 8 == 0, rows_per_group > 0,
 * rows % rows_per_group == 0 and eps >= 0. rows == 0 is a no-op. */
int dit_adaln_modulate(const void* x, const void* gamma, const void* beta, void* out,
                       int64_t rows, int32_t D, int64_t rows_per_group, float eps,
                       float scale_offset, void* stream);

/* Gated residual (DiT page, "A ruptura da U-Net"): out = x + alpha_g * y, alpha
 * a D-vector per group g = r / rows_per_group (a scalar gate is its broadcast;
 * alpha = 0 returns x exactly, the adaLN-Zero identity).
 *   x, y, out : [rows, D] bf16 (out may alias x or y);  alpha : [rows / rows_per_group, D] bf16
 * Errors: as dit_adaln_modulate. */
int dit_gated_residual(const void* x, const void* y, const void* alpha, void* out,
                       int64_t rows, int32_t D, int64_t rows_per_group, void* stream);

/* One Euler step of the rectified-flow sampler with per-frame local times (DiT
 * page, section "Flow Matching e Rectified Flow": straight path x_t = (1-t) x_0 +
 * t x_1, velocity u, 10-25 Euler or midpoint steps; "Flowception: Temporally
 * Expansive Flow Matching for Video Generation", section "Metodologia", interleaved
 * time schedule: each frame i has its own local time t_i):
 *   out[r, c] = x[r, c] + dt[g] * u[r, c],   g = r / rows_per_group
 * with dt[g] = t_g' - t_g the step of frame g (rows_per_group = tokens per frame).
 * fp32 FMA, one bf16 rounding; dt[g] == 0 returns x[r, :] bit for bit.
 *   x, u, out : [rows, D] bf16 (out may alias x: the in-place sampler update)
 *   dt        : [rows / rows_per_group] fp32, device memory, 4-byte aligned
 * Errors: as dit_adaln_modulate; DIT_ERR_NULL for a null pointer. */
int dit_flow_euler_step(const void* x, const void* u, const float* dt, void* out, int64_t rows,
                        int32_t D, int64_t rows_per_group, void* stream);

/* Linear layer of the block with fused epilogue (cost page, "Matematica por tras":
 * Y = X W; DiT page, "A ruptura da U-Net": the projections and the MLP inside the
 * adaLN-Zero residuals):
 *   y   = x w^T + bias                 x [M, K], w [N, K] (linear-layer [out, in] layout)
 *   y   = gelu(y) if activation == 1   tanh form y/2 (1 + tanh(sqrt(2/pi)(y + 0.044715 y^3)))
 *   out = residual + alpha[g] * y      if residual != NULL (g = row / rows_per_group;
 *                                      alpha[g, n] == 0 returns residual's bits), else y
 * bf16 in and out, fp32 accumulation in tensor memory, one bf16 rounding. bias [N]
 * may be NULL. residual [M, N] (may alias out), alpha [M / rows_per_group, N].
 * The GELU and the bias are this library's reading: the pages name only "MLP".
 * Errors: DIT_ERR_NULL (x, w, out, or alpha with residual); DIT_ERR_SHAPE unless
 * 0 <= M < 2^31, N > 0, K > 0, N % 8 == 0, K % 8 == 0, activation in {0, 1} and, with
 * a residual, rows_per_group > 0 dividing M; DIT_ERR_ALIGN for a pointer not 16-byte
 * aligned. M == 0 is a no-op. */
int dit_linear(const void* x, const void* w, const void* bias, void* out, int64_t M, int32_t N,
               int32_t K, int32_t activation, const void* residual, const void* alpha,
               int64_t rows_per_group, void* stream);

/* dit_linear on FP8 E4M3 operands (DiT page, "Engenharia de inferencia e paralelismo
 * de contexto: Ulysses, Ring Attention e FP8": weights and activations in FP8).
 * x8 [M, K] and w8 [N, K] are E4M3 codes standing for x_scale * x8 and w_scale * w8;
 * the products run as kind::f8f6f4 MMAs with fp32 accumulation, and the epilogue
 * (x_scale * w_scale, bias, GELU, gate) and every other argument are as in
 * dit_linear. K % 16 == 0. Errors: as dit_linear; DIT_ERR_SHAPE for a scale that is
 * not finite and positive. */
int dit_linear_fp8(const void* x8, const void* w8, const void* bias, void* out, int64_t M,
                   int32_t N, int32_t K, int32_t activation, const void* residual,
                   const void* alpha, int64_t rows_per_group, float x_scale, float w_scale,
                   void* stream);

/* Kernel form of dit_linear and dit_linear_fp8 for later calls in this process: 1
 * (default) runs CTA pairs (cta_group::2) on 256 x 256 tiles, each SM loading half of
 * every B tile, both CTAs' loads completing on the even CTA's barrier; 0 one CTA per
 * 128 x 256 tile. The two give the same bits; measured on B200 at the 480P projection
 * shapes the pair form is 8-15 % faster in bf16. No counterpart in the source pages. A
 * plain process-wide setting, not synchronised: set it before other threads issue
 * calls. Errors: DIT_ERR_SHAPE for any other value. */
int dit_set_linear_variant(int variant);

/* Standalone 3D-RoPE of q and k (DiT page, "3D-RoPE e atencao espaco-temporal"),
 * fp32 rotation of bf16 data, the same rotation for every head.
 *   q_in, k_in   : [rows, H, d] bf16; k_in may be NULL (then k_out is ignored)
 *   q_out, k_out : [rows, H, d] bf16; may equal q_in / k_in (in place)
 * Sequence layout: see the conventions above (positions restart per sequence).
 * Errors: DIT_ERR_SHAPE unless d is 64 or 128, H > 0, the bands are even and sum
 * to d, grid_h, grid_w >= 1, base > 1, offsets >= 0, and every sequence length
 * is a multiple of grid_h * grid_w; DIT_ERR_SEQLENS for a bad cu_seqlens. */
int dit_rope3d_qk(const void* q_in, const void* k_in, void* q_out, void* k_out, int64_t rows,
                  int32_t H, int32_t d, int32_t n_seq, const int32_t* cu_seqlens_dev,
                  const int32_t* cu_seqlens_host, const dit_rope3d_desc* rope, void* stream);

/* dit_rope3d_qk followed by E4M3 quantisation of its outputs, in one pass (DiT page,
 * "3D-RoPE e atencao espaco-temporal" for the rotation; "Engenharia de inferencia e
 * paralelismo de contexto: Ulysses, Ring Attention e FP8" for the FP8 operands):
 *   q8_out = e4m3(bf16(R3D q) * q_inv_scale),  k8_out = e4m3(bf16(R3D k) * k_inv_scale)
 * byte for byte what dit_rope3d_qk into bf16 buffers followed by dit_quantize_e4m3
 * of each gives, without writing and re-reading the rotated bf16 tensors: the
 * operands of dit_attn_fwd_qk8 / dit_attn_fwd_fp8.
 *   q_in, k_in     : [rows, H, d] bf16, 16-byte aligned; k_in may be NULL (k8_out
 *                    and k_inv_scale are then ignored)
 *   q8_out, k8_out : [rows, H, d] E4M3 codes, one byte each, 8-byte aligned; they
 *                    must overlap neither input nor each other (no in-place form)
 * Errors: as dit_rope3d_qk; DIT_ERR_SHAPE for an inverse scale that is not finite or
 * for overlapping buffers; DIT_ERR_ALIGN for misaligned pointers. */
int dit_rope3d_qk_e4m3(const void* q_in, const void* k_in, void* q8_out, void* k8_out,
                       int64_t rows, int32_t H, int32_t d, int32_t n_seq,
                       const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                       const dit_rope3d_desc* rope, float q_inv_scale, float k_inv_scale,
                       void* stream);

/* Full non-causal attention per sequence and head (DiT page, "3D-RoPE e atencao
 * espaco-temporal"; the Flowception summary: bidirectional attention over all
 * frames), flash-style on tcgen05 tensor cores: bf16 operands, fp32 scores,
 * fp32 online softmax and accumulation, bf16 output.
 *   o[i, h, :] = sum_j softmax_j(scale * <q_rot[i,h], k_rot[j,h]>) v[j, h, :]
 * over the keys j of the query's own sequence (packed sequences never see one
 * another). With `rope` non-NULL, q and k are rotated by 3D-RoPE inside the
 * kernel as their tiles are loaded (fp32 rotation, bf16 operand); with NULL they
 * are used as given. Rotating q and k first with dit_rope3d_qk and passing NULL
 * gives the same bits and is faster on long sequences (in-kernel, every K tile is
 * rotated again for each pair of query tiles); the in-kernel form needs no scratch.
 * Dense batches (cu_seqlens NULL) whose last wave of work units (a pair of 128-row
 * query tiles of one sequence and head, one CTA per SM) would leave most SMs idle run
 * that wave split by key range: each of those units is a cluster of 2-8 CTAs that
 * each take a share of the key tiles and merge their partial results through
 * distributed shared memory (no scratch memory). Such units differ from the unsplit
 * form only in rounding (the same online-softmax rescaling, applied across shares).
 *   q, k, v, o : [rows, H, d] bf16, o must not overlap q, k or v
 *   lse        : NULL or [rows, H] fp32, natural-log sum of exp(scale * scores)
 *   softmax_scale <= 0 selects 1/sqrt(d).
 * Errors: DIT_ERR_SHAPE unless d is 64 or 128, H > 0, rows > 0 ... (and, with
 * rope, as dit_rope3d_qk); DIT_ERR_SEQLENS for a bad cu_seqlens; DIT_ERR_DEVICE
 * off sm_100. */
int dit_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t rows,
                 int32_t H, int32_t d, int32_t n_seq, const int32_t* cu_seqlens_dev,
                 const int32_t* cu_seqlens_host, float softmax_scale, const dit_rope3d_desc* rope,
                 void* stream);

/* Allocation-free variant of dit_attn_fwd (no counterpart in the source pages).
 * Same arguments, layouts, results and errors as dit_attn_fwd; the difference is
 * where the 3D-RoPE cos/sin table lives. dit_attn_fwd allocates it with cudaMalloc
 * on first use and caches it; this call instead writes it (the same values, by the
 * same kernel) into a fixed array of device memory that belongs to the loaded library,
 * so it never calls cudaMalloc, cudaFree or any allocating routine. It is meant for
 * callers that must not allocate device memory while they run: processes that hand
 * all device memory to their own pool or allocator up front, memory-capped serving
 * workers, and latency-critical paths that cannot afford cudaMalloc's implicit
 * device synchronisation.
 *   - The array holds at most 65536 (cos, sin) pairs (512 KiB); a larger table (long
 *     videos or large patch grids) returns DIT_ERR_SCRATCH and launches nothing.
 *   - Every GPU that loads the library holds the array until the process exits. The
 *     driver places it when the library's device code is first loaded on a device,
 *     which is the first libdit3d call there (lazy loading): make any one libdit3d
 *     call on each device before handing the rest of its memory to a pool. If that
 *     load finds no memory, this call returns DIT_ERR_ALLOC.
 *   - The first call on a device looks up the array's device address (a runtime
 *     query, no allocation); make that first call before any stream capture.
 *     dit_shutdown() forgets the looked-up addresses.
 *   - All calls on a device share the one array, which keeps the last call's table:
 *     each call rewrites the whole range it uses (a fill kernel on `stream` before the
 *     attention), so calls on one stream are ordered, but calls whose work overlaps on
 *     the GPU (different streams without ordering) race on the array and must be
 *     serialised by the caller.
 *   - With rope == NULL no table is involved and the call is dit_attn_fwd exactly. */
int dit_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                         int64_t rows, int32_t H, int32_t d, int32_t n_seq,
                         const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                         float softmax_scale, const dit_rope3d_desc* rope, void* stream);

/* Attention whose Q K^T product runs on FP8 E4M3 operands (DiT page, "Engenharia de
 * inferencia e paralelismo de contexto: Ulysses, Ring Attention e FP8": E4M3/E5M2
 * activations). q8, k8: [rows, H, 128] E4M3 codes (one byte each, already rotated by
 * 3D-RoPE where wanted) standing for q_scale * q8 and k_scale * k8; v, o: [rows, H, 128]
 * bf16. Scores are softmax_scale * q_scale * k_scale * (q8 . k8) accumulated in fp32;
 * P and V stay bf16, exactly as in dit_attn_fwd. Sequences, lse and stream as in
 * dit_attn_fwd; no in-kernel RoPE. head_dim must be 128.
 * Errors: as dit_attn_fwd; DIT_ERR_SHAPE for d != 128 or a scale that is not finite
 * and positive. */
int dit_attn_fwd_qk8(const void* q8, const void* k8, const void* v, void* o, float* lse,
                     int64_t rows, int32_t H, int32_t d, int32_t n_seq,
                     const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                     float softmax_scale, float q_scale, float k_scale, void* stream);

/* Attention with E4M3 q, k and v (same page and section): S = q_scale k_scale (q8 . k8)
 * and O = v_scale (P8 . v8) / l both run as kind::f8f6f4 MMAs, with P rounded to E4M3
 * (P <= 2^8 by the lazy running maximum, inside E4M3's range) and the row sum l
 * accumulated from the unrounded fp32 P. q8, k8, v8: [rows, H, 128] E4M3 codes; o:
 * [rows, H, 128] bf16. Other arguments and errors as dit_attn_fwd_qk8. */
int dit_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse,
                     int64_t rows, int32_t H, int32_t d, int32_t n_seq,
                     const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                     float softmax_scale, float q_scale, float k_scale, float v_scale,
                     void* stream);

/* out8[i] = e4m3(x[i] * inv_scale): FP8 E4M3 codes of bf16 values, rounded to nearest
 * even and saturated at +-448 (same page and section). x: n bf16 (16-byte aligned),
 * out8: n bytes (8-byte aligned), n % 8 == 0. With inv_scale a power of two the
 * product is exact, so every code is the nearest E4M3 value of x * inv_scale.
 * Errors: DIT_ERR_NULL, DIT_ERR_SHAPE (n < 0, n % 8, inv_scale not finite),
 * DIT_ERR_ALIGN. n == 0 is a no-op. */
int dit_quantize_e4m3(const void* x, void* out8, int64_t n, float inv_scale, void* stream);

/* Waits for `stream`, then reads and clears the library's device error word.
 * Returns DIT_ERR_TIMEOUT if any kernel gave up a bounded wait since the last
 * check (its outputs are then invalid), DIT_ERR_LAUNCH on a CUDA error, else DIT_OK. */
int dit_check_device(void* stream);

/* Host watchdog form of dit_check_device: polls an event recorded on `stream` (no
 * blocking synchronisation) for at most timeout_us microseconds of wall time. Returns
 * DIT_ERR_TIMEOUT when the stream's work has not finished by then (the work keeps
 * running and the call may be repeated; this is how a host learns of a kernel that
 * stopped making progress without blocking on it), DIT_ERR_LAUNCH on a CUDA error;
 * once the stream has finished, reads and clears the device error word on that stream
 * and returns as dit_check_device does. DIT_ERR_SHAPE for a negative timeout. */
int dit_wait_device(void* stream, int64_t timeout_us);

/* Test hook of dit_wait_device's polling loop, with a fake query in place of the
 * event: the query reports "not yet" busy_polls times, then "done" (fail == 0) or
 * "failed" (fail != 0). Returns what dit_wait_device's loop returns (DIT_OK,
 * DIT_ERR_LAUNCH, DIT_ERR_TIMEOUT) and stores the number of polls made in *polls
 * (may be NULL). Needs no GPU. */
int dit_debug_poll_fake(int64_t busy_polls, int fail, int64_t timeout_us, int64_t* polls);

/* Test hook of the attention's FMA-pipe exponential (the share of the E4M3 modes'
 * softmax exponentials that does not run on the MUFU unit; no counterpart in the source
 * pages): out[i] = 2^t[i] by the kernel's own routine (round-to-nearest split t = j + f
 * with the 1.5 * 2^23 constant, degree-3 minimax polynomial for 2^f, j added to the
 * exponent field; t clamped to >= -126). t, out: device fp32 arrays of n elements; runs
 * on `stream`. Errors: DIT_ERR_SHAPE for n < 0, DIT_ERR_NULL for a null array when
 * n > 0, DIT_ERR_LAUNCH on a CUDA error. */
int dit_debug_exp2_fma(const float* t, float* out, int64_t n, void* stream);

/* Human-readable name of a dit_status code (static string, never NULL). */
const char* dit_status_string(int status);

/* Frees the cached RoPE tables of every device. Safe to call more than once. */
void dit_shutdown(void);

/* Selects the attention kernel for head_dim 128 (process-wide; head_dim 64 always
 * uses variant 0). 0 (default): one CTA per 256 query rows of a head on one SM.
 * 1: CTA pairs on two SMs sharing each tcgen05 MMA (cta_group::2, M = 256): each SM
 * loads and rotates half of every K tile and loads half of every V tile. Both give the
 * same results (same rounding steps); variant 0 is faster on the measured workloads.
 * A plain process-wide setting, not synchronised: set it before other threads issue
 * calls. The E4M3 attention calls always use variant 0.
 * Returns DIT_ERR_SHAPE for any other value. */
int dit_set_attn_variant(int variant);

/* Test hook: 1 makes the next attention launches give up their first wait at once
 * (exercising the bounded-wait error path without any hang), 0 restores. */
void dit_debug_force_timeout(int enable);

/* Test hook: the time limit, in nanoseconds, of the waits in later launches of the
 * single-CTA attention and linear kernels (0 restores the default of 2 s). A limit of
 * a few nanoseconds makes a wait that is not already satisfied run out: the kernel
 * leaves its work, drains its copies and MMAs and raises the error that the next
 * dit_check_device() returns as DIT_ERR_TIMEOUT. The CTA-pair kernels keep 2 s. A plain
 * process-wide setting, not synchronised. */
void dit_debug_wait_limit_ns(uint64_t ns);

/* Test hook: the number of CTAs each work unit of the last single-CTA attention launch
 * (dit_attn_fwd, dit_attn_fwd_noalloc, dit_attn_fwd_qk8, dit_attn_fwd_fp8 with
 * variant 0) was split over by key range: 1 for no split, 2-8 when a dense batch's last
 * partial wave ran as clusters that merge their partial results (see dit_attn_fwd), 0
 * before any launch. Not synchronised between threads. */
int dit_debug_last_attn_split(void);

/* Test hook of the split rule above, on the host with made-up figures (needs no GPU):
 * writes to *split the split S (1 = none) for `units` work units, `sms` SMs and `nk` key
 * tiles per unit, where resident[S] (S = 0..8) stands for the number of clusters of S
 * CTAs that fit at once: the largest S in 2..8 with (units % sms) * S <= sms,
 * 2 * S <= nk and resident[S] >= units % sms; 1 when units % sms == 0 or none
 * qualifies. Errors: DIT_ERR_NULL for a NULL `resident` or `split`. */
int dit_debug_tail_split(int64_t units, int64_t sms, int64_t nk, const int32_t* resident,
                         int32_t* split);

#ifdef __cplusplus
}
#endif

#endif /* DIT3D_H_ */
