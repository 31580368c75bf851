// NVFP4 block GEMMs for the Klein block: e2m1 operands (two values per
// byte), one e4m3 scale per 16 consecutive values along K, and an fp32
// second-level scale (one per weight matrix, one per activation row). The
// transformer's nvfp4 file (Diffusers release blog for FLUX.3 Image Klein,
// "Smaller GPUs, single files, and custom LoRA training"); NVFP4 runs on
// Blackwell tensor cores (local-run guide, quantised files).
//
// Quantisation (all decisions in fp32, each step one correctly rounded
// operation, in this order):
//   g     = amax / (448 * 6)                 (0 for an all-zero row / matrix)
//   s_b   = e4m3_rn_satfinite(amax_b / (6 * g))      per block of 16 values
//   code  = e2m1_rn_satfinite(x / (s_b * g))         (0 where s_b * g is 0)
//
// Layouts (device memory):
//   codes  [rows][cols / 2] bytes; value 2i of a row in the low 4 bits of
//          byte i, value 2i + 1 in the high 4 bits
//   scales 512-byte atoms: atom (R, C) holds rows 128R..128R+127 and columns
//          64C..64C+63 at byte (R * cols / 64 + C) * 512; in it, the scale of
//          row r and 16-value block b (0..3 within the 64 columns) sits at
//          (r % 32) * 16 + ((r % 128) / 32) * 4 + b. This is the order in
//          which tcgen05.cp (32x128b, warpx4) places scales in tensor memory
//          for the block-scaled MMA: lane r % 32 of each 32-lane group, 32-bit
//          column (r % 128) / 32, byte b. Rows past the matrix up to a
//          multiple of 128 hold scale 0.
//
// The GEMM (gemm_nvfp4_kernel) runs on CTA pairs: 256 x 128 output tiles
// (256 x 256, two N = 128 halves per A stage, for the out-projection),
// M = 256 from the two CTAs' 128 A rows, N = 128 from 64 B rows of each CTA;
// K in stages of 256 values (128 bytes per row, one 128-byte swizzle row);
// per stage each CTA also loads its A rows' scales (4 atoms) and the tile's
// B scales (4 atoms, the same in both CTAs). A scale warp copies them to the
// stage's slot in tensor memory and signals the MMA thread, which then
// issues the stage's four K = 64 MMAs
// (tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16). The copies
// run from their own thread because, queued by the MMA thread in front of
// the MMAs, they took about as long as the MMAs themselves. Tile
// configurations in nv::Cfg.
#include "common.cuh"
#include "internal.h"

namespace klein {

namespace nv {
// Tile configurations. Narrow (in-projection, plain GEMM): 256 x 128 tiles,
// two 128-column accumulators so that the epilogue of one tile overlaps the
// next, eight stages. Wide (out-projection): 256 x 256 tiles as two N = 128
// halves sharing each A stage, one 256-column accumulator, five stages; its
// epilogue is light next to 48 K stages a tile, so serialising it costs
// little, and each stage carries twice the MMA work per A byte.
template <bool WIDE>
struct Cfg {
  static constexpr int kHalves = WIDE ? 2 : 1;          // N = 128 halves per tile
  static constexpr int kStageA = 128 * 128;             // this CTA's 128 A rows x 128 bytes
  static constexpr int kStageB = kHalves * 64 * 128;    // this CTA's 64 B rows of each half
  static constexpr int kStageSFA = 4 * 512;             // four scale atoms (K = 256 values)
  static constexpr int kStageSFB = kHalves * 4 * 512;   // the same for each half's 128 B rows
  static constexpr int kStage = kStageA + kStageB + kStageSFA + kStageSFB;
  static constexpr int kStages = WIDE ? 5 : 8;
  static constexpr int kAccs = WIDE ? 1 : 2;
  static constexpr int kTileBytes = kStages * kStage;
  static constexpr int kSmem = kTileBytes + 1024 + 256;
  // TMEM: accumulators in columns 0..255, then one scale slot per smem
  // stage (A scales 16 columns, then 16 per half for B). The scale copies
  // come from a thread of their own, so nothing orders them after the MMAs
  // of earlier stages: giving every stage its own slot is what keeps a copy
  // from overwriting scales an MMA still reads.
  static constexpr uint32_t kSfCol0 = 256;
  static constexpr uint32_t kSfSlot = 16 + 16 * kHalves;
  static_assert(kAccs * 128 * kHalves == 256, "accumulators fill columns 0..255");
  static_assert(kSfCol0 + kStages * kSfSlot <= 512, "scale slots exceed the TMEM allocation");
  static_assert(kSmem <= 227 * 1024, "stages exceed shared memory");
  static_assert((3 * kStages + 5 + 1) * 8 + 4 <= 256, "barriers exceed their shared-memory area");
};
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiWarps = 8;
constexpr int kSfWarp = 2 + kEpiWarps;  // copies the block scales to tensor memory
constexpr int kThreads = 32 * (kSfWarp + 1);
constexpr float kG = 448.0f * 6.0f;
}  // namespace nv

// ------------------------------------------------------------------ element codes

// Two floats -> one byte of e2m1 codes (round to nearest even, saturating to
// +-6), `lo` in bits 0-3. cvt puts its first source in the upper half.
__device__ __forceinline__ uint32_t pack_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// e4m3 code of a non-negative float (round to nearest even, saturating).
__device__ __forceinline__ uint32_t e4m3_code(float x) { return pack_e4m3x4(x, 0.f, 0.f, 0.f) & 0xFFu; }

// Value of an e4m3 code (exact in fp32).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h2;
  const uint16_t c = static_cast<uint16_t>((code & 0xFFu) * 0x101u);  // the code in both bytes
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Byte offset of the scale of (row, 16-value block) in the atom layout.
__device__ __forceinline__ long long sf_offset(long long row, int block, int cols) {
  const long long atom = (row >> 7) * (cols >> 6) + (block >> 2);
  return atom * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (block & 3);
}

// Block scale and its step s_b * g for a 16-value block with maximum amax_b.
__device__ __forceinline__ void nvfp4_block_scale(float amax_b, float g, uint32_t& code, float& step) {
  if (g > 0.f) {
    code = e4m3_code(__fdiv_rn(amax_b, __fmul_rn(6.0f, g)));
    step = __fmul_rn(e4m3_value(code), g);
  } else {
    code = 0u;
    step = 0.f;
  }
}

__device__ __forceinline__ float nvfp4_div(float x, float step) { return step > 0.f ? __fdiv_rn(x, step) : 0.f; }

// ------------------------------------------------------------------ quantisers

// |x| maximum of a bf16 matrix into *amax_bits (float bits, non-negative
// values compare as integers); *amax_bits must start at 0.
__global__ void amax_kernel(const __nv_bfloat16* __restrict__ src, long long n, unsigned* amax_bits) {
  pdl_trigger();
  pdl_wait();
  float m = 0.f;
  const long long n8 = n >> 3;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const uint4 r = s4[i];
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = unpack_bf16(w[q]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// g = amax / 2688 in place (the bits of amax become the value g).
__global__ void tensor_scale_kernel(float* g) {
  pdl_trigger();
  pdl_wait();
  *g = __fdiv_rn(__uint_as_float(*reinterpret_cast<unsigned*>(g)), nv::kG);
}

// Source row of output row r of the in-projection weights in the NVFP4
// GEMM's tile order: q, k, v rows (0..9215) as they are, then for each
// 64-unit SwiGLU chunk c its 64 gate rows and its 64 up rows.
__device__ __forceinline__ long long in_proj_src_row(long long r) {
  if (r < 3 * kDim) return r;
  const long long c = (r - 3 * kDim) >> 7;
  const long long j = (r - 3 * kDim) & 127;
  return j < 64 ? 3 * kDim + 64 * c + j : 3 * kDim + kMlp + 64 * c + (j - 64);
}

// One CTA of 256 threads per row (at most 12288 columns, 8 bf16 per thread
// per chunk) of `batch` matrices of `rows` rows each, whose scales are laid
// out per matrix over rows_pad rows (CTA = b * rows_pad + r). With g_in NULL
// each row takes g = row amax / 2688, written to g_rows[b * rows + r];
// otherwise g = *g_in (the matrix's). in_proj_order: output rows in the
// in-projection's tile order (in_proj_src_row). The row is read whole before
// the block-wide max, so the codes may overwrite the row's own bytes
// (dst == src). Rows from `rows` to rows_pad write scale 0 only.
__global__ void __launch_bounds__(256) quantize_nvfp4_kernel(const __nv_bfloat16* src, long long src_ld,
                                                             int in_proj_order, uint8_t* dst, long long dst_ld,
                                                             uint8_t* __restrict__ sf, float* g_rows,
                                                             const float* __restrict__ g_in, int rows, int rows_pad,
                                                             int cols) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[8];
  const int b = blockIdx.x / rows_pad;
  const int r = blockIdx.x % rows_pad;
  const int nchunks = cols >> 3;
  if (r >= rows) {  // padding rows of the matrix's last atom row: scale 0
    for (int k = threadIdx.x; k < (cols >> 4); k += 256) sf[sf_offset(blockIdx.x, k, cols)] = 0;
    return;
  }
  const long long row = (long long)b * rows + r;
  const long long srow = in_proj_order ? in_proj_src_row(row) : row;
  const uint4* s4 = reinterpret_cast<const uint4*>(src + srow * src_ld);
  constexpr int kMaxChunks = 6;
  uint4 raw[kMaxChunks];
  float cmax[kMaxChunks];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxChunks; ++j) {
    const int c = threadIdx.x + 256 * j;
    raw[j] = c < nchunks ? s4[c] : make_uint4(0, 0, 0, 0);
    const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
    float m = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = unpack_bf16(w[q]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    cmax[j] = m;
    amax = fmaxf(amax, m);
  }
  float g;
  if (!g_in) {
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();  // every thread's loads of this row have returned
    amax = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    g = __fdiv_rn(amax, nv::kG);
    if (threadIdx.x == 0) g_rows[row] = g;
  } else {
    __syncthreads();  // the loads of this row have returned before any code is written over them
    g = *g_in;
  }
  uint32_t* d4 = reinterpret_cast<uint32_t*>(dst + row * dst_ld);
#pragma unroll
  for (int j = 0; j < kMaxChunks; ++j) {
    const int c = threadIdx.x + 256 * j;   // chunks c and c ^ 1 form one 16-value block
    const float bmax = fmaxf(cmax[j], __shfl_xor_sync(0xffffffffu, cmax[j], 1));
    if (c >= nchunks) continue;
    uint32_t code;
    float step;
    nvfp4_block_scale(bmax, g, code, step);
    const float2 f0 = unpack_bf16(raw[j].x), f1 = unpack_bf16(raw[j].y);
    const float2 f2 = unpack_bf16(raw[j].z), f3 = unpack_bf16(raw[j].w);
    d4[c] = pack_e2m1x2(nvfp4_div(f0.x, step), nvfp4_div(f0.y, step)) |
            (pack_e2m1x2(nvfp4_div(f1.x, step), nvfp4_div(f1.y, step)) << 8) |
            (pack_e2m1x2(nvfp4_div(f2.x, step), nvfp4_div(f2.y, step)) << 16) |
            (pack_e2m1x2(nvfp4_div(f3.x, step), nvfp4_div(f3.y, step)) << 24);
    if ((c & 1) == 0) sf[sf_offset(blockIdx.x, c >> 1, cols)] = static_cast<uint8_t>(code);
  }
}

// Modulated LayerNorm (as modln_kernel) with the output quantised to NVFP4,
// one second-level scale per row: one warp per row, the modulated row held in
// registers; lanes 4j..4j+3 hold one 16-value block for each t. The scales
// of each batch item are laid out over rows_pad rows (a multiple of 256, the
// GEMM's tile); warps of rows from `rows` to rows_pad write scale 0 only.
__global__ void __launch_bounds__(256, 1) modln_nvfp4_kernel(const float* __restrict__ x, long long x_bstride,
                                                          int x_row0, uint8_t* __restrict__ codes,
                                                          uint8_t* __restrict__ sf, float* __restrict__ g_rows,
                                                          int batch, int rows, int rows_pad, int n_txt, int n_img,
                                                          const float* __restrict__ mod, long long mod_stride) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= batch * rows_pad) return;
  const int b = warp / rows_pad;
  const int i = warp % rows_pad;
  uint8_t* sfb = sf + (long long)b * rows_pad * (kDim / 16);
  constexpr int kVec = kDim / 4 / 32;  // 24 float4 per lane
  if (i >= rows) {
    for (int t = 0; t < kVec; ++t)
      if ((lane & 3) == 0) sfb[sf_offset(i, 8 * t + (lane >> 2), kDim)] = 0;
    return;
  }
  const int grow = x_row0 + i;
  const float4* src = reinterpret_cast<const float4*>(x + ((long long)b * x_bstride + grow) * kDim);
  float4 v[kVec];
#pragma unroll
  for (int t = 0; t < kVec; ++t) v[t] = __ldg(src + lane + 32 * t);
  float sum = 0.f;
#pragma unroll
  for (int t = 0; t < kVec; ++t) sum += (v[t].x + v[t].y) + (v[t].z + v[t].w);
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum * (1.0f / kDim);
  float sq = 0.f;
#pragma unroll
  for (int t = 0; t < kVec; ++t) {
    const float a = v[t].x - mean, bb = v[t].y - mean, c = v[t].z - mean, d = v[t].w - mean;
    sq = fmaf(a, a, fmaf(bb, bb, fmaf(c, c, fmaf(d, d, sq))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = rsqrtf(sq * (1.0f / kDim) + 1e-6f);
  const int m = mode_of_row(grow, n_txt, n_img);
  const float4* shift = reinterpret_cast<const float4*>(mod + m * mod_stride);
  const float4* scl = reinterpret_cast<const float4*>(mod + m * mod_stride + kDim);
  float amax = 0.f;
#pragma unroll
  for (int t = 0; t < kVec; ++t) {
    const int c4 = lane + 32 * t;
    const float4 sc = __ldg(scl + c4);
    const float4 sh = __ldg(shift + c4);
    float4 e = v[t];
    e.x = fmaf((e.x - mean) * rstd, 1.f + sc.x, sh.x);
    e.y = fmaf((e.y - mean) * rstd, 1.f + sc.y, sh.y);
    e.z = fmaf((e.z - mean) * rstd, 1.f + sc.z, sh.z);
    e.w = fmaf((e.w - mean) * rstd, 1.f + sc.w, sh.w);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(e.x), fabsf(e.y)), fmaxf(fabsf(e.z), fabsf(e.w))));
    v[t] = e;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float g = __fdiv_rn(amax, nv::kG);
  const long long orow = (long long)b * rows + i;
  if (lane == 0) g_rows[orow] = g;
  uint16_t* dst = reinterpret_cast<uint16_t*>(codes + orow * (kDim / 2));
#pragma unroll
  for (int t = 0; t < kVec; ++t) {
    const float4 e = v[t];
    float bmax = fmaxf(fmaxf(fabsf(e.x), fabsf(e.y)), fmaxf(fabsf(e.z), fabsf(e.w)));
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 2));
    uint32_t code;
    float step;
    nvfp4_block_scale(bmax, g, code, step);
    dst[lane + 32 * t] = static_cast<uint16_t>(pack_e2m1x2(nvfp4_div(e.x, step), nvfp4_div(e.y, step)) |
                                               (pack_e2m1x2(nvfp4_div(e.z, step), nvfp4_div(e.w, step)) << 8));
    if ((lane & 3) == 0) sfb[sf_offset(i, 8 * t + (lane >> 2), kDim)] = static_cast<uint8_t>(code);
  }
}

int launch_quantize_nvfp4(const __nv_bfloat16* src, long long src_ld, int in_proj_order, uint8_t* dst,
                          long long dst_ld, uint8_t* sf, float* g_rows, float* g_matrix, int batch, int rows,
                          int rows_pad, int cols, cudaStream_t s) {
  if (rows <= 0 || batch <= 0) return 0;
  if (cols <= 0 || cols % 64 || cols > 12288 || rows_pad < rows || rows_pad % 128 ||
      (long long)batch * rows_pad > 0x7fffffffLL)
    return -2;
  const float* g_in = nullptr;
  if (g_matrix) {
    // the matrix's second-level scale: amax over every element, then / 2688
    // (a matrix, not a batch: src must be dense rows of `cols`)
    if (batch != 1 || src_ld != cols) return -2;
    if (cudaMemsetAsync(g_matrix, 0, sizeof(float), s) != cudaSuccess) return -1;
    const long long n = (long long)rows * cols;
    const int blocks = (int)((n / 8 + 255) / 256 < 4 * num_sms() ? (n / 8 + 255) / 256 : 4 * num_sms());
    cudaError_t e = launch_kernel(amax_kernel, dim3(blocks), dim3(256), 0, s, 1, src, n,
                                  reinterpret_cast<unsigned*>(g_matrix));
    note_launch();
    if (e != cudaSuccess) return -1;
    e = launch_kernel(tensor_scale_kernel, dim3(1), dim3(1), 0, s, 1, g_matrix);
    note_launch();
    if (e != cudaSuccess) return -1;
    g_in = g_matrix;
  }
  const cudaError_t e = launch_kernel(quantize_nvfp4_kernel, dim3((unsigned)((long long)batch * rows_pad)), dim3(256),
                                      0, s, 1, src, src_ld, in_proj_order, dst, dst_ld, sf, g_rows, g_in, rows,
                                      rows_pad, cols);
  note_launch();
  return (e == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

int launch_modln_nvfp4(const float* x, long long x_bstride, int x_row0, uint8_t* codes, uint8_t* sf, float* g_rows,
                       int batch, int rows, int n_txt, int n_img, const float* mod, long long mod_stride,
                       cudaStream_t s) {
  const int rows_pad = (rows + 255) / 256 * 256;  // the GEMM's 256-row tiles
  const long long warps = (long long)batch * rows_pad;
  if (warps <= 0) return 0;
  const cudaError_t e = launch_kernel(modln_nvfp4_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, 1, x,
                                      x_bstride, x_row0, codes, sf, g_rows, batch, rows, rows_pad, n_txt, n_img, mod,
                                      mod_stride);
  note_launch();
  return (e == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// ------------------------------------------------------------------ tensor core

// Instruction descriptor of kind::mxf4nvf4 with block scales: e2m1 A and B
// (format 1 in bits 7-9 and 10-12), both K-major, e4m3 scales (bit 23 = 0),
// scale byte 0 of each 32-bit TMEM column (bits 4-5 and 29-30 = 0), N >> 3 at
// bits 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_nvfp4(int m, int n) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// D (+)= (A * sfa) (B * sfb)^T over the pair: one 256 x N x 64 step.
__device__ __forceinline__ void umma_nvfp4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Copy of one 512-byte scale atom (32 rows of 16 bytes) from each CTA's
// shared memory into its tensor memory: four 32-bit columns, replicated in
// the four 32-lane groups.
__device__ __forceinline__ void tmem_cp_atom_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of a scale atom: K-major without swizzle, four
// 8-row x 16-byte core matrices 128 bytes apart (stride byte offset), one
// along K; version 1.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(128 >> 4) << 16) |
         (static_cast<uint64_t>(128 >> 4) << 32) | (static_cast<uint64_t>(1) << 46);
}

// ------------------------------------------------------------------ epilogues (128-column tiles)

// q or k head: RMS-normalise the head's 128 values, scale by the norm weight,
// rotate by RoPE; v head: stored transposed; SwiGLU tile: columns 0..63 gate,
// 64..127 up. part (0, 1): this warp's half of the columns (64 each; for q/k
// both halves take the sum of squares over all 128 columns).
__device__ __forceinline__ void nv_epi_qkv(uint32_t taddr, const GemmArgs& g, int b, int r, int n_idx, int part,
                                           float ga) {
  const bool valid = r < g.rows;
  const float sc = ga * __ldg(g.b_g);
  float v[32];
  if (n_idx < 72) {
    const int which = n_idx / 24;  // 0 q, 1 k, 2 v
    const int head = n_idx % 24;
    const long long bh = (long long)b * kHeads + head;
    if (which == 2) {
      __nv_bfloat16* dst = g.vt + bh * kHeadDim * g.rows_pad + r;
#pragma unroll 1
      for (int c = 2 * part; c < 2 * part + 2; ++c) {
        tmem_ld32(taddr + 32 * c, v);
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; ++i) dst[(long long)(32 * c + i) * g.rows_pad] = __float2bfloat16_rn(v[i] * sc);
        }
      }
      return;
    }
    const float* w = which == 0 ? g.q_norm : g.k_norm;
    __nv_bfloat16* dst = (which == 0 ? g.q : g.k) + (bh * g.rows_pad + r) * kHeadDim;
    float ss = 0.f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(taddr + 32 * c, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
    }
    // values are sc * acc: the scale folds into the normalisation
    const float rs = sc * rsqrtf(sc * sc * ss * (1.0f / kHeadDim) + 1e-6f);
    const float4* rope4 = reinterpret_cast<const float4*>(g.rope + (long long)(valid ? r : 0) * kPairs);
    const float4* w4 = reinterpret_cast<const float4*>(w);
#pragma unroll 1
    for (int c = 2 * part; c < 2 * part + 2; ++c) {
      tmem_ld32(taddr + 32 * c, v);
      if (!valid) continue;
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const int d = 32 * c + i;
        const float4 wn = __ldg(w4 + (d >> 2));
        const float4 cs = __ldg(rope4 + (d >> 2));
        const float y0 = v[i] * rs * wn.x, y1 = v[i + 1] * rs * wn.y;
        const float y2 = v[i + 2] * rs * wn.z, y3 = v[i + 3] * rs * wn.w;
        pk[i >> 1] = pack_bf16(y0 * cs.x - y1 * cs.y, y0 * cs.y + y1 * cs.x);
        pk[(i >> 1) + 1] = pack_bf16(y2 * cs.z - y3 * cs.w, y2 * cs.w + y3 * cs.z);
      }
      uint4* o = reinterpret_cast<uint4*>(dst + 32 * c);
      o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      o[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
      o[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
    }
  } else {
    const int chunk = n_idx - 72;  // hidden units 64 * chunk .. + 63
    __nv_bfloat16* dst = g.a_out + ((long long)b * g.rows + r) * kOutK + kDim + chunk * 64 + 32 * part;
    float u[32];
    tmem_ld32(taddr + 32 * part, v);
    tmem_ld32(taddr + 64 + 32 * part, u);
    if (!valid) return;
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2)
      pk[i >> 1] = pack_bf16(silu(v[i] * sc) * (u[i] * sc), silu(v[i + 1] * sc) * (u[i + 1] * sc));
    uint4* o = reinterpret_cast<uint4*>(dst);
    o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    o[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
    o[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
  }
}

// x += gate[mode(row)] * acc * scale over this warp's 64 of the tile's 128
// columns. Every lane takes part in the TMEM loads (warp-collective), rows
// past the end only skip the update.
__device__ __forceinline__ void nv_epi_resid(uint32_t taddr, const GemmArgs& g, int b, int r, int n_idx, int part,
                                             float ga) {
  const bool valid = r < g.rows;
  const float sc = ga * __ldg(g.b_g);
  const int grow = g.x_row0 + (valid ? r : 0);
  const int mode = mode_of_row(grow, g.n_txt, g.n_img);
  const float* gate = g.mod + (long long)mode * 3 * kDim + 2 * kDim + n_idx * 128;
  float* xr = g.x + ((long long)b * g.x_bstride + grow) * kDim + n_idx * 128;
  float v[32];
#pragma unroll 1
  for (int c = 2 * part; c < 2 * part + 2; ++c) {
    tmem_ld32(taddr + 32 * c, v);
    if (!valid) continue;
    float4* p = reinterpret_cast<float4*>(xr + 32 * c);
    const float4* gt = reinterpret_cast<const float4*>(gate + 32 * c);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 xv = p[i];
      const float4 gv = __ldg(gt + i);
      xv.x = fmaf(gv.x, v[4 * i + 0] * sc, xv.x);
      xv.y = fmaf(gv.y, v[4 * i + 1] * sc, xv.y);
      xv.z = fmaf(gv.z, v[4 * i + 2] * sc, xv.z);
      xv.w = fmaf(gv.w, v[4 * i + 3] * sc, xv.w);
      p[i] = xv;
    }
  }
}

// out (fp32) = acc * scale over this warp's 64 columns.
__device__ __forceinline__ void nv_epi_store(uint32_t taddr, const GemmArgs& g, int b, int r, int n_idx, int part,
                                             float ga) {
  const bool valid = r < g.rows;
  const float sc = ga * __ldg(g.b_g);
  float v[32];
#pragma unroll 1
  for (int c = 2 * part; c < 2 * part + 2; ++c) {
    tmem_ld32(taddr + 32 * c, v);
    if (!valid) continue;
    float* o = reinterpret_cast<float*>(g.out) + ((long long)b * g.out_bstride + g.out_row0 + r) * g.out_ld +
               n_idx * 128 + 32 * c;
#pragma unroll
    for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(o + i) = make_float4(v[i] * sc, v[i + 1] * sc, v[i + 2] * sc, v[i + 3] * sc);
  }
}

// ------------------------------------------------------------------ the GEMM

template <int EPI>
__global__ void __launch_bounds__(nv::kThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                      const GemmArgs g) {
  using C = nv::Cfg<EPI == kEpiResid>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kTileBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* sf_ready = empty + C::kStages;  // [kStages]: the stage's scales are in tensor memory
  uint64_t* acc_full = sf_ready + C::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* sf_drain = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * 32 * nv::kEpiWarps);
    }
    mbar_init(drain, 1);
    mbar_init(sf_drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    tma_prefetch_desc(&map_sfa);
    tma_prefetch_desc(&map_sfb);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, nv::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // operands and outputs are touched only after the previous kernel completes

  // g.n_tiles counts 128-column tiles; a wide tile covers kHalves of them
  const int n_tiles = g.n_tiles / C::kHalves;
  const int m_tiles = g.batch * g.m_tiles_per_b;
  const int total = m_tiles * n_tiles;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  constexpr uint32_t idesc = idesc_nvfp4(256, 128);
  const int k_atoms = g.k_blocks * 4;  // 64-value scale columns along K

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      StageLog log;
      for (int tile = pair; tile < total; tile += npairs) {
        const int m_idx = g.n_fastest ? tile / n_tiles : tile % m_tiles;
        const int n_idx = g.n_fastest ? tile % n_tiles : tile / m_tiles;
        const int b = m_idx / g.m_tiles_per_b;
        const int mt = m_idx % g.m_tiles_per_b;
        const int row0 = mt * 256 + 128 * static_cast<int>(rank);
        // scale atoms: this CTA's 128 A rows (atom row 2 mt + rank of batch
        // item b), and each half's 128 B rows (atom row of that half)
        const int sfa_row = (b * g.m_tiles_per_b * 2 + 2 * mt + static_cast<int>(rank)) * k_atoms;
        bool ok = true;
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, 0x131)) { ok = false; break; }
          if (leader) {
            mbar_arrive_expect_tx(&full[stage], 2 * C::kStage);
            log.armed(stage, phase);
          }
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
          uint8_t* sa = smem + stage * C::kStage;
          uint8_t* ssfa = sa + C::kStageA + C::kStageB;
          tma_load_3d_pair(sa, &map_a, bar, kb * 128, row0, b);
          tma_load_2d_pair(ssfa, &map_sfa, bar, 0, sfa_row + 4 * kb);
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) {
            const int n128 = n_idx * C::kHalves + h;
            tma_load_2d_pair(sa + C::kStageA + h * 64 * 128, &map_b, bar, kb * 128,
                             n128 * 128 + 64 * static_cast<int>(rank));
            tma_load_2d_pair(ssfa + C::kStageSFA + h * 4 * 512, &map_sfb, bar, 0, n128 * k_atoms + 4 * kb);
          }
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
      if (leader) log.drain(full, C::kStages, 0x135);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int tile = pair; tile < total; tile += npairs, ++it) {
        const int acc = C::kAccs == 2 ? (it & 1) : 0;
        const uint32_t acc_phase = C::kAccs == 2 ? ((it >> 1) & 1) : (it & 1);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, 0x132)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * 128;
        bool ok = true;
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          // operands in shared memory, and their scales in the stage's
          // tensor-memory slot (copied by the scale warp)
          if (!mbar_wait(&full[stage], phase, 0x133) || !mbar_wait(&sf_ready[stage], phase, 0x137)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::kStage);
          const uint32_t b0 = a0 + C::kStageA;
          const uint32_t sfa_t = tmem_base + C::kSfCol0 + C::kSfSlot * stage;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h)
              umma_nvfp4_pair(d + 128 * h, sw128_desc(a0 + 32 * k), sw128_desc(b0 + h * 64 * 128 + 32 * k), idesc,
                              sfa_t + 4 * k, sfa_t + 16 + 16 * h + 4 * k, (kb | k) != 0);
          }
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair(&acc_full[acc], 0x3);
      }
      umma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, 0x136);
    }
  } else if (warp == nv::kSfWarp) {
    // Block scales to tensor memory, from a thread of their own: issued by
    // the MMA thread, each stage's copies sat in its tensor-core queue ahead
    // of the MMAs and cost about as much time as the MMAs. The copy for
    // stage s of step n lands in slot s, which the MMAs of step n - kStages
    // last read; those completed before the producer could refill stage s,
    // which this thread waited for.
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      const int steps = ((total - pair + npairs - 1) / npairs) * g.k_blocks;
      for (int n = 0; n < steps; ++n) {
        if (!mbar_wait(&full[stage], phase, 0x138)) break;
        tc_fence_after();
        const uint32_t sfa0 = smem_u32(smem + stage * C::kStage) + C::kStageA + C::kStageB;
        const uint32_t sfa_t = tmem_base + C::kSfCol0 + C::kSfSlot * stage;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          tmem_cp_atom_pair(sfa_t + 4 * k, sf_atom_desc(sfa0 + 512 * k));
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h)
            tmem_cp_atom_pair(sfa_t + 16 + 16 * h + 4 * k, sf_atom_desc(sfa0 + C::kStageSFA + h * 4 * 512 + 512 * k));
        }
        umma_commit_pair(&sf_ready[stage], 0x1);
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
      // every copy issued here has completed before tensor memory is freed
      umma_commit_pair(sf_drain, 0x1);
      mbar_wait(sf_drain, 0, 0x139);
    }
  } else {
    const int quarter = warp & 3;
    const int rloc = quarter * 32 + lane;
    const int part = (warp - 2) / 4;
    int it = 0;
    for (int tile = pair; tile < total; tile += npairs, ++it) {
      const int m_idx = g.n_fastest ? tile / n_tiles : tile % m_tiles;
      const int n_idx = g.n_fastest ? tile % n_tiles : tile / m_tiles;
      const int b = m_idx / g.m_tiles_per_b;
      const int r = (m_idx % g.m_tiles_per_b) * 256 + 128 * static_cast<int>(rank) + rloc;
      const int acc = C::kAccs == 2 ? (it & 1) : 0;
      const uint32_t acc_phase = C::kAccs == 2 ? ((it >> 1) & 1) : (it & 1);
      if (!mbar_wait(&acc_full[acc], acc_phase, 0x134)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + acc * 128 + (static_cast<uint32_t>(quarter * 32) << 16);
      const float ga = r < g.rows ? __ldg(g.a_scale + (long long)b * g.rows + r) : 0.f;
#pragma unroll 1
      for (int h = 0; h < C::kHalves; ++h) {
        const int n128 = n_idx * C::kHalves + h;  // the 128-column tile this half covers
        if (EPI == kEpiF32) nv_epi_store(taddr + 128 * h, g, b, r, n128, part, ga);
        else if (EPI == kEpiQKV) nv_epi_qkv(taddr + 128 * h, g, b, r, n128, part, ga);
        else nv_epi_resid(taddr + 128 * h, g, b, r, n128, part, ga);
      }
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[acc]), 0));
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, nv::kTmemCols);
  }
}

template <int EPI>
static int launch_nvfp4_one(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& msfa,
                            const CUtensorMap& msfb, const GemmArgs& g, cudaStream_t s) {
  using C = nv::Cfg<EPI == kEpiResid>;
  if (g.n_tiles % C::kHalves != 0) return -3;  // a wide tile covers two 128-column tiles
  static int max_pairs_dev[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return -1;
  int& max_pairs = max_pairs_dev[dev];
  if (max_pairs == 0) {
    if (cudaFuncSetAttribute(gemm_nvfp4_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
        cudaSuccess)
      return -1;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    cfg.blockDim = dim3(nv::kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_kernel<EPI>, &cfg) != cudaSuccess || n < 1) return -1;
    max_pairs = n;
  }
  const int total = g.batch * g.m_tiles_per_b * (g.n_tiles / C::kHalves);
  if (total <= 0) return 0;
  const int pairs = total < max_pairs ? total : max_pairs;
  const cudaError_t e = launch_kernel(gemm_nvfp4_kernel<EPI>, dim3(2 * pairs), dim3(nv::kThreads), C::kSmem, s, 2,
                                      ma, mb, msfa, msfb, g);
  note_launch();
  return (e == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// Scale atoms viewed as a 2-D array of 32-bit words [atoms][128]; a box of
// 4 atoms (2 KB) per load, no swizzle.
static int make_map_sf(CUtensorMap* map, const void* sf, long long atoms) {
  return make_map_2d_u32(map, sf, 128, (uint64_t)atoms, 512, 128, 4);
}

int launch_gemm_nvfp4(int epi, const void* a, long long a_ld, const void* a_sf, const void* b, const void* b_sf,
                      const GemmArgs& g, int n_rows_b, cudaStream_t s) {
  // A: [batch][rows] rows of K/2 bytes at pitch a_ld bytes; B: [n_rows_b][K/2] bytes
  const int kbytes = g.k_blocks * 128;
  const long long a_atoms = (long long)g.batch * g.m_tiles_per_b * 2 * g.k_blocks * 4;
  const long long b_atoms = (long long)(n_rows_b / 128) * g.k_blocks * 4;
  CUtensorMap ma, mb, msfa, msfb;
  if (make_map_3d(&ma, a, kbytes, g.rows, g.batch, a_ld, (uint64_t)g.rows * a_ld, 128, 128, 1) ||
      make_map_2d(&mb, b, kbytes, n_rows_b, kbytes, 128, 64, 1) || make_map_sf(&msfa, a_sf, a_atoms) ||
      make_map_sf(&msfb, b_sf, b_atoms))
    return -2;
  switch (epi) {
    case kEpiF32: return launch_nvfp4_one<kEpiF32>(ma, mb, msfa, msfb, g, s);
    case kEpiQKV: return launch_nvfp4_one<kEpiQKV>(ma, mb, msfa, msfb, g, s);
    case kEpiResid: return launch_nvfp4_one<kEpiResid>(ma, mb, msfa, msfb, g, s);
  }
  return -2;
}

}  // namespace klein
