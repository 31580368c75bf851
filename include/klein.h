/*
 * klein.h - C ABI of the B200 (sm_100a) implementation of the FLUX.3 Image
 * Klein denoiser hot path: the joint transformer block over the concatenated
 * [text | noisy image | reference] token sequence, run inside the shifted
 * flow-matching Euler loop.
 *
 * Sources (cited by page and section):
 *   [blog]   "FLUX.3 Image Klein Is Now Available in Diffusers", section
 *            "Speed, architecture, and how the tokens move" (two stages,
 *            block shape, modulation by stream, RoPE axes).
 *   [blogzh] its Chinese translation: block pseudo-code and RoPE table.
 *   [guide]  "How to Run FLUX 3 Image Klein Locally": "The latent space and
 *            the VAE", "Inside the transformer", "The denoise loop", "What
 *            step distillation removed", "Why dropping CFG halves the compute".
 *
 * Conventions for every call:
 *   - Pointers marked "device" are caller-owned CUDA device memory; the
 *     library borrows them for the duration of the asynchronous work it
 *     enqueues and never frees them. "host" pointers are read or written
 *     before the call returns.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream).
 *   - Argument errors are detected synchronously and return a negative
 *     klein_status with nothing enqueued; klein_last_error() then returns a
 *     message (thread-local, valid until the next call on that thread).
 *   - A failed kernel launch returns KLEIN_ERR_CUDA. A device-side wait that
 *     gave up (no progress for the wait limit) is recorded on the device and
 *     reported by klein_sync(stream) or klein_device_status() as
 *     KLEIN_ERR_TIMEOUT.
 *   - Device pointers must be 16-byte aligned. The model width is fixed at
 *     KLEIN_DIM = 3072, 24 heads of 128.
 *   - bf16 = IEEE bfloat16 stored as uint16; all matrices are row-major.
 *   - Nothing is thrown across the ABI; no call allocates device memory:
 *     scratch comes from the caller's workspace.
 */
#ifndef KLEIN_H
#define KLEIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KLEIN_DIM 3072
#define KLEIN_HEADS 24
#define KLEIN_HEAD_DIM 128
#define KLEIN_MLP_HIDDEN 9216
#define KLEIN_LATENT_CH 128
#define KLEIN_MAX_REFS 10
#define KLEIN_IN_COLS (3 * KLEIN_DIM + 2 * KLEIN_MLP_HIDDEN)  /* 27648 */
#define KLEIN_OUT_K (KLEIN_DIM + KLEIN_MLP_HIDDEN)            /* 12288 */

typedef enum {
  KLEIN_OK = 0,
  KLEIN_ERR_INVALID_ARG = -1,
  KLEIN_ERR_SHAPE = -2,
  KLEIN_ERR_ALIGN = -3,
  KLEIN_ERR_WORKSPACE = -4,
  KLEIN_ERR_CUDA = -5,
  KLEIN_ERR_TIMEOUT = -6,
  KLEIN_ERR_UNSUPPORTED = -7
} klein_status;

/* Message describing the last error on this thread ("" if none). */
const char* klein_last_error(void);

/* ABI version (major * 100 + minor). */
int klein_version(void);

/* Number of kernels this library has launched in this process (host-side
 * counter over every entry point; for launch accounting in benchmarks). */
long long klein_launch_count(void);

/* Reads and clears the device error word on the current device (blocking:
 * synchronises the device). Returns KLEIN_OK, KLEIN_ERR_TIMEOUT when a
 * bounded wait gave up, KLEIN_ERR_CUDA on a CUDA error. `site` (may be NULL)
 * receives the code of the wait that gave up. */
int klein_device_status(unsigned* site);

/* Waits for the work queued on `stream`, then reports as klein_device_status
 * does (without synchronising other streams): KLEIN_OK, KLEIN_ERR_TIMEOUT when
 * a bounded wait gave up, KLEIN_ERR_CUDA on a CUDA error. The device error
 * word is per device: a wait that gave up in this library's work on another
 * stream of the same device is reported (and cleared) here too. */
int klein_sync(void* stream);

/* Sets the bound (nanoseconds) of every device-side wait; default 2 s. */
int klein_set_wait_limit_ns(unsigned long long ns);

/* Enqueues a probe kernel that waits, with the given bound, on a barrier
 * that nothing arrives on. It must end by recording KLEIN_ERR_TIMEOUT, which
 * klein_device_status() then returns. Tests the wait bound, nothing else. */
int klein_wait_probe(unsigned long long limit_ns, void* stream);

/* Launch profiler. While running, the library records a pair of CUDA
 * events on the launching stream around each kernel launch of the path and
 * tags it with its kind (index into the arrays below):
 *   0 modulated LayerNorm, 1 in-projection GEMM (QKV + MLP-in, fused
 *   epilogue), 2 attention, 3 out-projection GEMM (gated residual) of
 *   blocks over a whole sequence (the joint blocks);
 *   4 timestep embedding + modulation, 5 input / output projections,
 *   6 Euler update, 7 other, 8 rowwise e4m3 quantisation of the
 *   out-projection's input (FP8 blocks only);
 *   9, 10, 11, 12: kinds 0..3 of blocks over a row range of the sequence
 *   (the stage-1 blocks, one stream each).
 * klein_profile_begin(max_launches) creates the events (host-side
 * resources; no device memory); klein_profile_end synchronises, writes the
 * summed milliseconds and launch counts per kind (arrays of
 * KLEIN_PROF_KINDS, either may be NULL) and releases the events. Returns
 * KLEIN_ERR_WORKSPACE if more launches happened than max_launches (those
 * were not timed). Not thread-safe; one profile at a time. */
#define KLEIN_PROF_KINDS 13
int klein_profile_begin(int max_launches);
int klein_profile_end(double* ms, int* launches);

/* ------------------------------------------------------------------ sequence */

/* Token layout of one denoiser call: rows [0, n_txt) text, then the image
 * grid img_h x img_w scanned row-major, then each reference grid in order
 * ([blog]: the sequence is [text | image | reference]). A 1024x1024 image
 * is a 64 x 64 grid of 4096 tokens ([guide] "The latent space and the VAE"). */
typedef struct {
  int batch;                    /* B: 1, or 2 for guidance (cond, uncond) */
  int n_txt;                    /* text tokens per batch item (>= 1) */
  int img_h, img_w;             /* image token grid */
  int n_refs;                   /* reference images, 0..KLEIN_MAX_REFS */
  int ref_h[KLEIN_MAX_REFS];    /* reference token grids */
  int ref_w[KLEIN_MAX_REFS];
} klein_seq;

/* Token counts of `seq`; any output pointer may be NULL. */
int klein_seq_tokens(const klein_seq* seq, int* n_img, int* n_ref, int* n_total);

/* Text length padded to a multiple of 80 ([blog]; [guide] "The text
 * encoder"). A helper: the kernels accept any n_txt. Returns -1 if n < 0. */
int klein_pad_text_len(int n);

/* Shifted sigma schedule ([guide] "The denoise loop"): `steps` levels evenly
 * spaced from 1 down to 1/steps, each mapped to s*sigma/(1+(s-1)*sigma),
 * then a final 0. sigmas: host, steps + 1 floats. Computed in double. */
int klein_sigma_schedule(int steps, float shift, float* sigmas);

/* (t, h, w, l) per token ([blogzh] RoPE table; Chinese summary page for
 * the negative reference offset): text i -> (0,0,0,i); image token (r,c)
 * -> (0,r,c,0); token (r,c) of reference k -> (0,r,c,-(k+1)).
 * pos: device, [n_total][4] float. */
int klein_positions(const klein_seq* seq, float* pos, void* stream);

/* ------------------------------------------------------------------ block */

/* Weights of one block (device, borrowed):
 *   w_in   bf16 [27648][3072]: output rows q(3072) | k(3072) | v(3072) |
 *          gate(9216) | up(9216); the SwiGLU hidden is silu(gate) * up.
 *   w_out  bf16 [3072][12288]: input columns attention (3072, the attention
 *          output projection) | MLP down (9216).
 *   q_norm, k_norm  float [128]: QK-RMSNorm weights shared by all heads.
 *   w_in_scale, w_out_scale  NULL for a bf16 block. Both set: the block is
 *          rowwise FP8 (the transformer's "fp8r" file, Diffusers release
 *          blog, "Smaller GPUs, single files, and custom LoRA training"):
 *          w_in and w_out then hold e4m3 codes (one byte per element, same
 *          shapes) and w_in_scale float [27648], w_out_scale float [3072]
 *          one scale per output row, as klein_quantize_rowwise_e4m3 writes
 *          them. The block quantises its two GEMM inputs (the modulated
 *          LayerNorm rows, and the [attention | SwiGLU] rows) the same way
 *          per token and runs both GEMMs on e4m3 tensor cores with fp32
 *          accumulation; everything else is as in the bf16 block.
 *   w_in_sf, w_out_sf  NULL unless the block is NVFP4 (the transformer's
 *          nvfp4 file, same blog section; NVFP4 runs on Blackwell tensor
 *          cores, "How to Run FLUX 3 Image Klein Locally"). Both set: w_in
 *          and w_out hold e2m1 codes as klein_quantize_nvfp4 writes them
 *          (w_in [27648][1536] bytes in the in-projection order of
 *          KLEIN_NVFP4_IN_PROJ, w_out [3072][6144]), w_in_sf / w_out_sf their
 *          block scales, and w_in_scale / w_out_scale each point to ONE float,
 *          the matrix's second-level scale. The block quantises its two GEMM
 *          inputs to NVFP4 per token (one second-level scale per row) and runs
 *          both GEMMs on the block-scaled fp4 tensor cores with fp32
 *          accumulation; attention and everything else stay as in the bf16
 *          block. */
typedef struct {
  const void* w_in;
  const void* w_out;
  const float* q_norm;
  const float* k_norm;
  const float* w_in_scale;
  const float* w_out_scale;
  const void* w_in_sf;
  const void* w_out_sf;
} klein_block_weights;

/* NVFP4 quantisation of a bf16 matrix src [rows][cols] (row pitch cols):
 * e2m1 values (1 sign, 2 exponent bits with bias 1, 1 mantissa bit;
 * magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), one e4m3 scale per 16 consecutive
 * values of a row, and fp32 second-level scales. All decisions in fp32, each
 * step one correctly rounded operation: g = amax / 2688 (0 if all zero);
 * block scale s = e4m3_rn_satfinite(amax_block / (6 g)); code =
 * e2m1_rn_satfinite(x / (s g)), 0 where s g = 0.
 *   mode   KLEIN_NVFP4_MATRIX: one g for the matrix (amax over all of it),
 *          written to g[0]; KLEIN_NVFP4_ROWS: one g per row (g[rows]);
 *          KLEIN_NVFP4_IN_PROJ: as MATRIX for a block's w_in [27648][3072],
 *          with the output rows in the NVFP4 in-projection's order: q, k, v
 *          rows (0..9215) as they are, then for each 64-unit chunk c of the
 *          SwiGLU hidden its gate rows 64c..64c+63 and its up rows 64c..64c+63.
 *   codes  device [rows][cols / 2] bytes; value 2i in the low 4 bits of byte i
 *   sf     device, round_up(rows, P) * cols / 16 bytes, P = 256 in ROWS mode
 *          and 128 otherwise: 512-byte atoms, atom (R, C) for rows
 *          128R..128R+127 and columns 64C..64C+63 at byte (R * cols / 64 + C)
 *          * 512, the scale of row r, block b (0..3 in the atom's 64 columns)
 *          at (r % 32) * 16 + ((r % 128) / 32) * 4 + b; padding rows get 0.
 *          This is the order in which the tensor core reads block scales.
 * cols a multiple of 64, at most 12288; codes must not overlap src.
 * Errors: KLEIN_ERR_SHAPE, KLEIN_ERR_ALIGN, KLEIN_ERR_INVALID_ARG. */
#define KLEIN_NVFP4_MATRIX 0
#define KLEIN_NVFP4_ROWS 1
#define KLEIN_NVFP4_IN_PROJ 2
int klein_quantize_nvfp4(const void* src, long long rows, int cols, int mode, void* codes, void* sf, float* g,
                         void* stream);

/* Rowwise e4m3 quantisation of a bf16 matrix src [rows][cols] (row pitch
 * cols): codes [rows][cols] bytes, scale [rows] float. Per row, in fp32:
 * amax = max |x|, inv = 448 / amax and scale = amax / 448 (correctly rounded
 * divisions), code = e4m3(x * inv) rounded to nearest even and saturated to
 * +-448 (OCP 8-bit floating point, E4M3: bias 7, no infinities); an all-zero
 * row gets scale 0 and codes 0. This is how FP8 block weights are made
 * (klein_block_weights). cols a multiple of 8, at most 12288; pointers
 * 16-byte aligned; codes must not overlap src. Errors: KLEIN_ERR_SHAPE,
 * KLEIN_ERR_ALIGN, KLEIN_ERR_INVALID_ARG. */
int klein_quantize_rowwise_e4m3(const void* src, long long rows, int cols, void* codes, float* scale,
                                void* stream);

/* Workspace bytes for klein_block_forward on `rows` rows of `batch` items. */
size_t klein_block_workspace_size(int batch, int rows);

/* One block, in place on rows [row0, row0 + rows) of every batch item of x
 * ([blogzh] block pseudo-code; [blog]; [guide] "Inside the transformer"):
 * no-affine LayerNorm modulated per stream (text rows use mode 0, image
 * rows mode 1, reference rows mode 2, by global row index against n_txt
 * and n_txt + n_img); q, k, v and the SwiGLU MLP from that one normalised
 * input; RMSNorm + 4-axis RoPE on q and k; softmax attention among the
 * `rows` rows only, no mask; x += gate * (attention out-projection + MLP).
 * A joint block passes row0 = 0, rows = n_total; a stage-1 block passes one
 * stream's row range (each stream attends only to itself).
 *   x        device float [batch][n_total][3072] (the residual stream is
 *            kept in fp32), updated in place
 *   pos      device float [n_total][4] (klein_positions)
 *   mod      device float [3 modes][3 (shift, scale, gate)][3072]
 *   ws       device workspace, >= klein_block_workspace_size(batch, rows)
 * Errors: KLEIN_ERR_SHAPE if rows < 1, the range leaves [0, n_total), a
 * stream size is negative or n_txt + n_img > n_total. */
int klein_block_forward(const klein_block_weights* w, void* x, int batch, int n_total, int row0, int rows,
                        int n_txt, int n_img, const float* pos, const float* mod, void* ws, size_t ws_bytes,
                        void* stream);

/* klein_block_forward without a workspace. The pages have no counterpart:
 * this entry point exists for callers that cannot call cudaMalloc, such as
 * a plug-in inside a host application that owns all device memory through
 * its own pool and forbids allocating around it, or code on a
 * latency-critical path where a device allocation (which may synchronise
 * the device) is not allowed. Same arguments and results as
 * klein_block_forward, minus ws / ws_bytes.
 *   - Scratch lives in one fixed array of this library's device memory
 *     (about 12.1 MiB), held on every GPU that loads the library until the
 *     process exits. It fits batch * round_up(rows, 128) <= 256; larger
 *     calls return KLEIN_ERR_WORKSPACE and enqueue nothing.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - Every call shares the one array and it keeps the last call's
 *     contents; nothing in it needs to start at zero (every value read is
 *     written earlier in the same call). Calls that overlap on the GPU (on
 *     different streams, or from several threads) race on it: serialise them.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
int klein_block_forward_static(const klein_block_weights* w, void* x, int batch, int n_total, int row0, int rows,
                               int n_txt, int n_img, const float* pos, const float* mod, void* stream);

/* ------------------------------------------------------------------ model */

/* All weights of a stack (device, borrowed; bf16 [out][in] unless noted).
 * Model: n_stage1 = 5 per-stream blocks and n_joint = 28 joint blocks
 * ([blog]; [guide] "Inside the transformer"); smaller counts are accepted. */
typedef struct {
  int n_stage1;
  int n_joint;
  const klein_block_weights* stage1[3];  /* per stream (txt, img, ref): n_stage1 each */
  const klein_block_weights* joint;      /* n_joint */
  const void* img_in;      /* [3072][128] image latent projection */
  const void* ref_in;      /* [3072][128] reference latent projection (may be NULL without refs) */
  const void* t_mlp1;      /* [3072][256] timestep embedder, layer 1 */
  const void* t_mlp2;      /* [3072][3072] layer 2 */
  const void* tt_mlp1;     /* target-level embedder of the distilled model, or NULL (base) */
  const void* tt_mlp2;
  const void* mod[2][3];   /* [9216][3072] per stage (1, 2) and stream: (shift, scale, gate) */
  const void* final_mod;   /* [6144][3072] final (shift, scale) */
  const void* final_out;   /* [128][3072] output projection to latent channels */
  const void* txt_in;      /* [3072][20480] text input projection, or NULL. The text encoder's
                              hidden states from eight of its layers, 2560 wide each, stacked to
                              20480 per token ([blog]; [guide] "The text encoder"), are projected to
                              the model width. NULL: text is given already at 3072. */
} klein_model_desc;

typedef struct klein_model klein_model;

/* Copies the descriptor (not the weights) into a new handle. */
int klein_model_create(klein_model** out, const klein_model_desc* desc);
void klein_model_destroy(klein_model* m);

/* Workspace bytes for klein_stack_forward / klein_denoise on `seq`. A
 * workspace serves one call at a time: calls that overlap on the device
 * (different streams) need their own. klein_denoise keeps state in it across
 * its steps (the projected text; for the base model, the text and reference
 * streams' stage-1 output, computed at the first step and reused after it). */
size_t klein_stack_workspace_size(const klein_seq* seq);

/* One denoiser call ([blog]; [guide] "Inside the transformer", "What step
 * distillation removed"): modulation from the timestep embedding (image
 * rows at sigma, text and reference rows at 0, plus the target-level
 * embedding of sigma_next on every stream when the model is distilled);
 * image and reference latents projected to 3072; stage 1 runs each stream's
 * own blocks over its own rows; stage 2 runs the joint blocks over
 * [text | image | reference]; the image rows then pass the final modulated
 * LayerNorm and projection to 128 channels.
 *   latents  device float [n_img][128], shared by the batch
 *   text     device bf16 [batch][n_txt][3072], or [batch][n_txt][20480] (the
 *            stacked encoder layers) when the model has txt_in; the
 *            projection runs once per klein_denoise call (text does not
 *            change across steps)
 *   refs     device float [n_ref][128] or NULL when seq->n_refs == 0
 *   v_out    device float [batch][n_img][128]
 *   ws       device workspace >= klein_stack_workspace_size(seq) */
int klein_stack_forward(const klein_model* m, const float* latents, const void* text, const float* refs,
                        float sigma, float sigma_next, const klein_seq* seq, float* v_out, void* ws,
                        size_t ws_bytes, void* stream);

/* Flow-matching Euler sampler ([guide] "The denoise loop", "Why dropping CFG
 * halves the compute"): from sigma = 1 over klein_sigma_schedule(steps,
 * shift), each step runs klein_stack_forward and moves the latents by
 * (sigma_next - sigma) * v. cfg > 1 needs seq->batch == 2 (text = cond then
 * uncond) and uses v = v_u + cfg (v_c - v_u); otherwise seq->batch == 1.
 *   latents  device float [n_img][128]: in = noise, out = the final latents
 *   x0_out   device float or NULL: the x0 preview x0 = x - sigma v of a step,
 *            taken before that step's update ([guide] "The denoise loop";
 *            [blogzh] Modular Diffusers preview block, a preview after every
 *            denoiser call): with x0_every_step = 0, [n_img][128] receives the
 *            last step's; otherwise [steps][n_img][128] receives every step's */
int klein_denoise(const klein_model* m, float* latents, const void* text, const float* refs, int steps,
                  float cfg, float shift, const klein_seq* seq, float* x0_out, int x0_every_step, void* ws,
                  size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ single ops
 * The kernels of the path, exposed one by one for parity tests and the
 * memory-bound benchmarks. Same conventions as above. */

/* h = modulated LayerNorm of rows [row0, row0 + rows) of x (mode by global
 * row as in klein_block_forward). mod: [3][>=2][3072] with per-mode stride
 * mod_stride floats; single_mode != 0 applies mod[0] to every row.
 * x: float [batch][n_total][3072]; h: bf16 [batch][rows][3072]. */
int klein_op_modln(const void* x, int batch, int n_total, int row0, int rows, int n_txt, int n_img,
                   const float* mod, long long mod_stride, int single_mode, void* h, void* stream);

/* cos/sin table [rows][64] (float2) of the 4-axis RoPE, theta = base. */
int klein_op_rope_table(const float* pos, int rows, float theta, void* table, void* stream);

/* out = RoPE(in) for bf16 [rows][heads][128] using a table from
 * klein_op_rope_table (in and out may alias). */
int klein_op_rope(const void* in, void* out, const void* table, int rows, int heads, void* stream);

/* x += dsigma * v with v = v_cond, or v_u + g (v_c - v_u) when v_uncond is
 * not NULL; x0_out (optional) = x - sigma * v, from x before the update.
 * float arrays of n elements, n a multiple of 4. */
int klein_op_euler(float* x, const float* v_cond, const float* v_uncond, long long n, float dsigma, float g,
                   float* x0_out, float sigma, void* stream);

/* C[M][N] (float) = A[M][K] * B[N][K]^T, bf16 operands, tcgen05 tensor cores.
 * M >= 1, N a multiple of 128, K a multiple of 64. */
int klein_op_gemm(const void* a, const void* b, float* c, int m, int n, int k, void* stream);

/* C[m][n] (float) = a_scale[m] * b_scale[n] * sum_k A[m][k] * B[n][k], A and
 * B e4m3 codes (bytes, row pitch K), on the e4m3 tensor-core GEMM of the FP8
 * block. M >= 1, N a multiple of 256, K a multiple of 128. */
int klein_op_gemm_e4m3(const void* a, const float* a_scale, const void* b, const float* b_scale, float* c, int m,
                       int n, int k, void* stream);

/* klein_op_modln with the output quantised rowwise to e4m3, as the FP8
 * block's first step does: codes [batch][rows][3072] bytes, scale
 * [batch][rows] float (the rule of klein_quantize_rowwise_e4m3, applied to
 * the fp32 normalised rows). Per-stream modes as in klein_block_forward. */
int klein_op_modln_e4m3(const void* x, int batch, int n_total, int row0, int rows, int n_txt, int n_img,
                        const float* mod, long long mod_stride, void* codes, float* scale, void* stream);

/* klein_op_modln with the output quantised to NVFP4 as the NVFP4 block's
 * first step does (KLEIN_NVFP4_ROWS rule on the fp32 normalised rows):
 * codes [batch][rows][1536] bytes, sf per batch item over round_up(rows, 256)
 * rows (the layout of klein_quantize_nvfp4; batch item b at b *
 * round_up(rows, 256) * 192 bytes), g [batch][rows]. */
int klein_op_modln_nvfp4(const void* x, int batch, int n_total, int row0, int rows, int n_txt, int n_img,
                         const float* mod, long long mod_stride, void* codes, void* sf, float* g, void* stream);

/* C[m][n] (float) = a_g[row] * (*b_g) * sum_k (A code * A block scale)
 * (B code * B block scale) on the block-scaled fp4 tensor cores of the NVFP4
 * block. A: codes [m][k/2] with scales over round_up(m, 256) rows and a_g
 * [m] (klein_quantize_nvfp4 in ROWS mode); B: codes [n][k/2] with scales and
 * one b_g (MATRIX mode). M >= 1, N a multiple of 128, K a multiple of 256. */
int klein_op_gemm_nvfp4(const void* a, const void* a_sf, const float* a_g, const void* b, const void* b_sf,
                        const float* b_g, float* c, int m, int n, int k, void* stream);

/* Softmax attention per (batch, head) over `rows` rows, scale 1/sqrt(128),
 * no mask. q, k: bf16 [batch][24][rows_pad][128]; vt: bf16
 * [batch][24][128][rows_pad] (v transposed); out: bf16 [batch][rows][out_ld]
 * with head h in columns h*128..h*128+127. rows_pad >= rows, a multiple of 8. */
int klein_op_attention(const void* q, const void* k, const void* vt, int batch, int rows, int rows_pad,
                       void* out, long long out_ld, void* stream);

/* Per-stage, per-stream modulation and the final (shift, scale) of one
 * denoiser call (see klein_stack_forward). mod_out: device float
 * [2][3][3][3072]; final_out: device float [2][3072]; ws: device,
 * >= 24576 floats (8 x 3072). */
int klein_op_time_mod(const klein_model* m, float sigma, float sigma_next, int with_ref, float* mod_out,
                      float* final_out, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KLEIN_H */
