// Internal (C++) interface between the Klein kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace klein {

// ------------------------------------------------------------------ TMA maps

// 2-D bf16 tensor map over a row-major [outer][inner] matrix with row pitch
// `row_bytes`; box = box_inner x box_outer elements, 128-byte swizzle.
// bytes1 = 1: one-byte elements (e4m3 codes) instead of bf16.
int make_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                uint32_t box_inner, uint32_t box_outer, int bytes1 = 0);
// 3-D bf16 tensor map over [d2][d1][d0] with byte strides s1 (d1) and s2 (d2).
int make_map_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                uint64_t s2, uint32_t box0, uint32_t box1, int bytes1 = 0);
// 2-D map of 32-bit words [outer][inner], no swizzle (dense boxes).
int make_map_2d_u32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer);

// ------------------------------------------------------------------ GEMM

enum EpiKind : int {
  kEpiF32 = 0,    // out fp32 = acc
  kEpiBF16 = 1,   // out bf16 = acc (optionally replicated over batch copies)
  kEpiQKV = 2,    // fused in-projection: RMSNorm + RoPE on q/k, v transposed, SwiGLU
  kEpiResid = 3,  // x += gate[mode(row)] * acc
};

struct GemmArgs {
  int batch;          // batch items of A (3-D map depth)
  int rows;           // valid rows of A per batch item (M)
  int m_tiles_per_b;  // ceil(rows / 128)
  int n_tiles;        // N / BN
  int k_blocks;       // K / 64
  int b_split;        // kEpiQKV: the N-tile where the paired gate|up tiles begin
  int n_fastest;      // visit tiles N-fastest (B fits in L2, A streamed once) instead of M-fastest
  // kEpiF32 / kEpiBF16: out[(b * out_bstride + out_row0 + r) * out_ld + n]
  void* out;
  long long out_ld;
  long long out_bstride;
  int out_row0;
  int replicate;      // >1: A has one batch item; write its rows into this many batch copies
  // kEpiQKV
  __nv_bfloat16* q;   // [batch][24][rows_pad][128]
  __nv_bfloat16* k;   // [batch][24][rows_pad][128]
  __nv_bfloat16* vt;  // [batch][24][128][rows_pad]
  __nv_bfloat16* a_out;  // [batch][rows][12288]; SwiGLU goes to columns 3072..
  const float* q_norm;
  const float* k_norm;
  const float2* rope;  // [rows][64] (cos, sin)
  int rows_pad;
  // kEpiResid
  float* x;           // residual stream, fp32 [batch][x_bstride rows][3072]
  long long x_bstride;
  int x_row0;
  const float* mod;   // [3 modes][3][3072] (shift, scale, gate)
  int n_txt, n_img;
  // e4m3 operands (launch_gemm_pair with e4m3 = 1): acc * a_scale[b * rows + r] * b_scale[B row]
  const float* a_scale;
  const float* b_scale;
  // NVFP4 operands (launch_gemm_nvfp4): acc * a_scale[b * rows + r] * (*b_g)
  const float* b_g;
};

// C[M,N] = A[M,K] * B[N,K]^T with epilogue `epi`; bn = 128 or 256.
// Same product on CTA pairs (clusters of 2) with 256 x 256 tiles: args.m_tiles_per_b
// counts 256-row tiles, args.n_tiles 256-column tiles; epi is kEpiF32, kEpiQKV or kEpiResid.
// With e4m3 = 1 both operands are rowwise-scaled e4m3 codes (maps of bytes,
// 128-byte boxes) and k_blocks counts 128-element K blocks; epi is kEpiQKV or
// kEpiResid.
int launch_gemm_pair(int epi, const CUtensorMap& map_a, const CUtensorMap& map_b, const GemmArgs& args,
                     cudaStream_t stream, int e4m3 = 0);
int launch_gemm(int bn, int epi, const CUtensorMap& map_a, const CUtensorMap& map_b, const GemmArgs& args,
                cudaStream_t stream);

// NVFP4 GEMM on CTA pairs (256 x 128 tiles; args.m_tiles_per_b counts 256-row
// tiles, n_tiles 128-column tiles, k_blocks 256-value K blocks): A codes
// [batch][rows][K/2] with scale atoms over round_up(rows, 256) rows per batch
// item, B codes [n_rows_b][K/2] with scale atoms (n_rows_b a multiple of
// 128); epi is kEpiF32, kEpiQKV (tile n < 72: head n % 24 of q, k, v; else
// 64 SwiGLU hidden units, B rows 64 gate then 64 up) or kEpiResid (256 x 256
// tiles: n_tiles must be even). Returns 0, -1 (launch), -2 (tensor map) or
// -3 (shape).
int launch_gemm_nvfp4(int epi, const void* a, long long a_ld, const void* a_sf, const void* b, const void* b_sf,
                      const GemmArgs& args, int n_rows_b, cudaStream_t stream);
// NVFP4 quantisation of `batch` bf16 matrices [rows][cols] (see nvfp4.cu);
// g_matrix: one scale for the whole (single) matrix, computed here;
// otherwise one per row into g_rows. in_proj_order: the in-projection
// weights' rows in the NVFP4 GEMM's tile order.
int launch_quantize_nvfp4(const __nv_bfloat16* src, long long src_ld, int in_proj_order, uint8_t* dst,
                          long long dst_ld, uint8_t* sf, float* g_rows, float* g_matrix, int batch, int rows,
                          int rows_pad, int cols, cudaStream_t stream);
int launch_modln_nvfp4(const float* x, long long x_bstride, int x_row0, uint8_t* codes, uint8_t* sf, float* g_rows,
                       int batch, int rows, int n_txt, int n_img, const float* mod, long long mod_stride,
                       cudaStream_t stream);

// ------------------------------------------------------------------ attention

struct AttnArgs {
  int batch, heads, rows, rows_pad;
  const __nv_bfloat16* q;   // [batch][heads][rows_pad][128]
  const __nv_bfloat16* k;   // [batch][heads][rows_pad][128]
  const __nv_bfloat16* vt;  // [batch][heads][128][rows_pad]
  __nv_bfloat16* out;       // [batch][rows][out_ld], head h at columns h*128..
  long long out_ld;
  float scale_log2;         // log2(e) / sqrt(128)
};

// Builds the operand tensor maps and launches the attention kernel.
// Returns 0, -1 on a launch error, -2 if a tensor map cannot be encoded.
int launch_attention(const AttnArgs& args, cudaStream_t stream);

// ------------------------------------------------------------------ memory-bound kernels

int launch_modln(const float* x, long long x_bstride, int x_row0, __nv_bfloat16* h, int batch, int rows,
                 int n_txt, int n_img, const float* mod, long long mod_mode_stride, int single_mode,
                 cudaStream_t stream);
// Same normalisation and modulation, output quantised rowwise to e4m3:
// codes [batch][rows][3072] bytes and one fp32 scale per row ([batch][rows]).
int launch_modln_e4m3(const float* x, long long x_bstride, int x_row0, uint8_t* codes, float* scale, int batch,
                      int rows, int n_txt, int n_img, const float* mod, long long mod_mode_stride,
                      cudaStream_t stream);
// Rowwise e4m3 quantisation of bf16 rows: src row r at src + r * src_ld
// (elements), codes of row r at dst + r * dst_ld (bytes), scale[r]. cols a
// multiple of 8, at most 12288. dst may alias src when dst_ld >= cols and
// dst_ld <= 2 * src_ld (each row is read whole before it is written).
int launch_quantize_rows(const __nv_bfloat16* src, long long src_ld, uint8_t* dst, long long dst_ld, float* scale,
                         long long rows, int cols, cudaStream_t stream);
int launch_rope_table(const float* pos, float2* table, int rows, float theta, cudaStream_t stream);
int launch_rope_apply(const __nv_bfloat16* in, __nv_bfloat16* out, const float2* table, int rows, int heads,
                      cudaStream_t stream);
int launch_positions(float* pos, int n_txt, int img_h, int img_w, int n_refs, const int* ref_h,
                     const int* ref_w, cudaStream_t stream);
int launch_euler(float* x, const float* v_cond, const float* v_uncond, long long n, float dsigma, float g,
                 float* x0_out, float sigma, cudaStream_t stream);
int launch_to_bf16(const float* in, __nv_bfloat16* out, long long n, cudaStream_t stream);
int launch_rows_to_f32(const __nv_bfloat16* src, long long src_bstride, float* dst, long long dst_bstride,
                       int dst_row0, int batch, int rows, cudaStream_t stream);

// Timestep embedding + modulation (a2).
struct TimeModArgs {
  const __nv_bfloat16* t_mlp1;  // [3072][256]
  const __nv_bfloat16* t_mlp2;  // [3072][3072]
  const __nv_bfloat16* tt_mlp1; // distilled target-time embedder, or null
  const __nv_bfloat16* tt_mlp2;
  const __nv_bfloat16* mod[2][3];  // [9216][3072]
  const __nv_bfloat16* final_mod;  // [6144][3072]
  float sigma, sigma_next;
  int with_ref;
  float* scratch;       // >= 8 * 3072 floats
  float* mod_out;       // [2][3][3][3072]
  float* final_out;     // [2][3072]
};
int launch_time_mod(const TimeModArgs& a, cudaStream_t stream);
int launch_gemv(const __nv_bfloat16* w, int n_out, int k, const float* x, int n_vec, long long x_stride,
                float* y, long long y_stride, int act_in_silu, const float* add, cudaStream_t stream);

int launch_wait_probe(unsigned long long limit_ns, cudaStream_t stream);
int num_sms();
// Index of the current device, or -1 if it is outside [0, kMaxDevices).
// Per-function launch settings (shared-memory opt-in, cluster occupancy) are
// per device, so the launchers keep them per device index.
constexpr int kMaxDevices = 64;
int current_device();

// Host-side count of kernels launched by this library (all entry points).
void note_launch();

}  // namespace klein
