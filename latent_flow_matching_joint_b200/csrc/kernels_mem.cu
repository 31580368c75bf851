// HBM-bound and small kernels of the Klein hot path: modulated LayerNorm,
// RoPE table and standalone rotation, token positions, Euler/CFG update,
// bf16 conversion, timestep embedding and the modulation GEMVs.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace klein {

// ------------------------------------------------------------------ modLN
// Parameter-free LayerNorm of each row, then (1 + scale[m]) * xhat + shift[m]
// with m the row's stream (Diffusers release blog for FLUX.3 Klein, "Speed,
// architecture, and how the tokens move": no learned affine; text and
// reference rows take the t = 0 modulation, image rows the current t).
// The residual stream x is fp32; h is the bf16 A operand of the
// in-projection. One warp per row: 24 x 16-byte loads per lane, fp32
// statistics (two passes over registers), 8-byte bf16 stores.

__global__ void __launch_bounds__(256, 2) modln_kernel(const float* __restrict__ x, long long x_bstride,
                                                    int x_row0, __nv_bfloat16* __restrict__ h, int batch,
                                                    int rows, int n_txt, int n_img,
                                                    const float* __restrict__ mod, long long mod_stride,
                                                    int single_mode) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= batch * rows) return;
  const int b = warp / rows;
  const int i = warp % rows;
  const int grow = x_row0 + i;
  const float4* src = reinterpret_cast<const float4*>(x + ((long long)b * x_bstride + grow) * kDim);
  uint2* dst = reinterpret_cast<uint2*>(h + ((long long)b * rows + i) * kDim);
  constexpr int kVec = kDim / 4 / 32;  // 24 float4 per lane
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
  const int m = single_mode ? 0 : mode_of_row(grow, n_txt, n_img);
  const float4* shift = reinterpret_cast<const float4*>(mod + m * mod_stride);
  const float4* scale = reinterpret_cast<const float4*>(mod + m * mod_stride + kDim);
#pragma unroll
  for (int t = 0; t < kVec; ++t) {
    const int c4 = lane + 32 * t;
    const float4 sc = __ldg(scale + c4);
    const float4 sh = __ldg(shift + c4);
    const float4 e = v[t];
    dst[c4] = make_uint2(pack_bf16(fmaf((e.x - mean) * rstd, 1.f + sc.x, sh.x), fmaf((e.y - mean) * rstd, 1.f + sc.y, sh.y)),
                         pack_bf16(fmaf((e.z - mean) * rstd, 1.f + sc.z, sh.z), fmaf((e.w - mean) * rstd, 1.f + sc.w, sh.w)));
  }
}

int launch_modln(const float* x, long long x_bstride, int x_row0, __nv_bfloat16* h, int batch, int rows,
                 int n_txt, int n_img, const float* mod, long long mod_stride, int single_mode, cudaStream_t s) {
  const long long warps = (long long)batch * rows;
  if (warps <= 0) return 0;
  const int blocks = (int)((warps + 7) / 8);
  const cudaError_t le = launch_kernel(modln_kernel, dim3(blocks), dim3(256), 0, s, 1, x, x_bstride, x_row0, h, batch, rows, n_txt, n_img, mod, mod_stride,
                                      single_mode);
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// ---- rowwise e4m3 quantisation (the transformer's rowwise FP8 weights,
// Diffusers release blog for FLUX.3 Image Klein, "Smaller GPUs, single files,
// and custom LoRA training"). Decision in fp32: amax = max |x| over the row,
// inv = 448 / amax and scale = amax / 448 (correctly rounded divisions),
// code = e4m3_rn_satfinite(x * inv); an all-zero row has scale 0.

__device__ __forceinline__ void e4m3_row_scales(float amax, float& inv, float& scale) {
  inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
  scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 0.f;
}

// modLN with the output quantised: one warp per row, as modln_kernel. The
// modulated row stays in registers between the row maximum and the codes
// (two blocks of 8 warps per SM; at 128 registers ptxas spills 28 bytes of
// the row, and the kernel is still faster than at one block per SM because
// twice the loads are in flight).
__global__ void __launch_bounds__(256, 2) modln_e4m3_kernel(const float* __restrict__ x, long long x_bstride,
                                                         int x_row0, uint32_t* __restrict__ codes,
                                                         float* __restrict__ scale, int batch, int rows,
                                                         int n_txt, int n_img, const float* __restrict__ mod,
                                                         long long mod_stride) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= batch * rows) return;
  const int b = warp / rows;
  const int i = warp % rows;
  const int grow = x_row0 + i;
  const float4* src = reinterpret_cast<const float4*>(x + ((long long)b * x_bstride + grow) * kDim);
  uint32_t* dst = codes + ((long long)b * rows + i) * (kDim / 4);
  constexpr int kVec = kDim / 4 / 32;
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
  float inv, s;
  e4m3_row_scales(amax, inv, s);
#pragma unroll
  for (int t = 0; t < kVec; ++t) {
    const float4 e = v[t];
    dst[lane + 32 * t] = pack_e4m3x4(__fmul_rn(e.x, inv), __fmul_rn(e.y, inv), __fmul_rn(e.z, inv), __fmul_rn(e.w, inv));
  }
  if (lane == 0) scale[(long long)b * rows + i] = s;
}

int launch_modln_e4m3(const float* x, long long x_bstride, int x_row0, uint8_t* codes, float* scale, int batch,
                      int rows, int n_txt, int n_img, const float* mod, long long mod_stride, cudaStream_t s) {
  const long long warps = (long long)batch * rows;
  if (warps <= 0) return 0;
  const int blocks = (int)((warps + 7) / 8);
  const cudaError_t le = launch_kernel(modln_e4m3_kernel, dim3(blocks), dim3(256), 0, s, 1, x, x_bstride, x_row0, reinterpret_cast<uint32_t*>(codes), scale, batch,
                                           rows, n_txt, n_img, mod, mod_stride);
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// One CTA of 256 threads per row; 8 bf16 per thread per chunk, at most 6
// chunks (12288 columns). The whole row is in registers before the block-wide
// max, so codes may overwrite the row's own source bytes.
constexpr int kQuantMaxChunks = 6;

__global__ void __launch_bounds__(256) quantize_rows_kernel(const __nv_bfloat16* src, long long src_ld,
                                                            uint8_t* dst, long long dst_ld,
                                                            float* __restrict__ scale, int cols) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[8];
  const long long row = blockIdx.x;
  const int nchunks = cols >> 3;
  const uint4* s4 = reinterpret_cast<const uint4*>(src + row * src_ld);
  uint4 raw[kQuantMaxChunks];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < kQuantMaxChunks; ++j) {
    const int c = threadIdx.x + 256 * j;
    raw[j] = c < nchunks ? s4[c] : make_uint4(0, 0, 0, 0);
    const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = unpack_bf16(w[q]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();  // every thread's loads of this row have returned
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  float inv, s;
  e4m3_row_scales(amax, inv, s);
  uint2* d2 = reinterpret_cast<uint2*>(dst + row * dst_ld);
#pragma unroll
  for (int j = 0; j < kQuantMaxChunks; ++j) {
    const int c = threadIdx.x + 256 * j;
    if (c >= nchunks) break;
    const float2 f0 = unpack_bf16(raw[j].x), f1 = unpack_bf16(raw[j].y);
    const float2 f2 = unpack_bf16(raw[j].z), f3 = unpack_bf16(raw[j].w);
    d2[c] = make_uint2(pack_e4m3x4(__fmul_rn(f0.x, inv), __fmul_rn(f0.y, inv), __fmul_rn(f1.x, inv), __fmul_rn(f1.y, inv)),
                       pack_e4m3x4(__fmul_rn(f2.x, inv), __fmul_rn(f2.y, inv), __fmul_rn(f3.x, inv), __fmul_rn(f3.y, inv)));
  }
  if (threadIdx.x == 0) scale[row] = s;
}

int launch_quantize_rows(const __nv_bfloat16* src, long long src_ld, uint8_t* dst, long long dst_ld, float* scale,
                         long long rows, int cols, cudaStream_t s) {
  if (rows <= 0) return 0;
  if (cols <= 0 || cols % 8 || cols > 256 * 8 * kQuantMaxChunks || rows > 0x7fffffffLL) return -2;
  const cudaError_t le = launch_kernel(quantize_rows_kernel, dim3((unsigned)rows), dim3(256), 0, s, 1, src, src_ld, dst, dst_ld, scale, cols);
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// bf16 rows -> fp32 rows of the residual stream: src [batch][rows][3072]
// (batch stride src_bstride rows) into dst rows [dst_row0, dst_row0 + rows)
// of each batch item (batch stride dst_bstride rows).
__global__ void rows_to_f32_kernel(const uint4* __restrict__ src, long long src_bstride, float4* __restrict__ dst,
                                   long long dst_bstride, int dst_row0, int rows, long long total) {
  pdl_trigger();
  pdl_wait();
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  constexpr int kPerRow = kDim / 8;
  const long long row = idx / kPerRow;
  const int c = static_cast<int>(idx % kPerRow);
  const long long b = row / rows;
  const long long r = row % rows;
  const uint4 raw = __ldg(src + (b * src_bstride + r) * kPerRow + c);
  const float2 a = unpack_bf16(raw.x), bb = unpack_bf16(raw.y), cc = unpack_bf16(raw.z), d = unpack_bf16(raw.w);
  float4* o = dst + ((b * dst_bstride + dst_row0 + r) * kPerRow + c) * 2;
  o[0] = make_float4(a.x, a.y, bb.x, bb.y);
  o[1] = make_float4(cc.x, cc.y, d.x, d.y);
}

int launch_rows_to_f32(const __nv_bfloat16* src, long long src_bstride, float* dst, long long dst_bstride,
                       int dst_row0, int batch, int rows, cudaStream_t s) {
  const long long total = (long long)batch * rows * (kDim / 8);
  if (total <= 0) return 0;
  const cudaError_t le = launch_kernel(rows_to_f32_kernel, dim3((int)((total + 255) / 256)), dim3(256), 0, s, 1, reinterpret_cast<const uint4*>(src), src_bstride,
                                                                  reinterpret_cast<float4*>(dst), dst_bstride,
                                                                  dst_row0, rows, total);
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// ------------------------------------------------------------------ RoPE
// Four axes (t, h, w, l), 32 head dims each (blog, RoPE paragraph); pair p =
// 16 * axis + j covers dims (2p, 2p+1) and turns by pos[axis] * theta^(-j/16).
// The table is built in double precision once per sequence.

__global__ void rope_table_kernel(const float* __restrict__ pos, float2* __restrict__ table, int rows,
                                  double theta) {
  pdl_trigger();
  pdl_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * kPairs) return;
  const int r = idx / kPairs;
  const int p = idx % kPairs;
  const int axis = p >> 4;
  const int j = p & 15;
  const double freq = pow(theta, -static_cast<double>(j) / 16.0);
  const double ang = static_cast<double>(pos[r * 4 + axis]) * freq;
  double sn, cs;
  sincos(ang, &sn, &cs);
  table[idx] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
}

int launch_rope_table(const float* pos, float2* table, int rows, float theta, cudaStream_t s) {
  const int n = rows * kPairs;
  if (n <= 0) return 0;
  const cudaError_t le = launch_kernel(rope_table_kernel, dim3((n + 255) / 256), dim3(256), 0, s, 1, pos, table, rows, static_cast<double>(theta));
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// Standalone rotation of [rows][heads][128] bf16 (the same arithmetic as the
// in-projection epilogue). One thread per 8 elements (4 pairs).
__global__ void rope_apply_kernel(const uint4* __restrict__ in, uint4* __restrict__ out,
                                  const float2* __restrict__ table, int rows, int heads) {
  pdl_trigger();
  pdl_wait();
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)rows * heads * (kHeadDim / 8);
  if (idx >= total) return;
  const int chunk = static_cast<int>(idx % (kHeadDim / 8));
  const int r = static_cast<int>(idx / ((long long)heads * (kHeadDim / 8)));
  const uint4 raw = __ldcs(in + idx);
  const float4* tp = reinterpret_cast<const float4*>(table + (long long)r * kPairs + chunk * 4);
  const float4 t01 = __ldg(tp);
  const float4 t23 = __ldg(tp + 1);
  const float2 e0 = unpack_bf16(raw.x), e1 = unpack_bf16(raw.y), e2 = unpack_bf16(raw.z), e3 = unpack_bf16(raw.w);
  uint4 o;
  o.x = pack_bf16(e0.x * t01.x - e0.y * t01.y, e0.x * t01.y + e0.y * t01.x);
  o.y = pack_bf16(e1.x * t01.z - e1.y * t01.w, e1.x * t01.w + e1.y * t01.z);
  o.z = pack_bf16(e2.x * t23.x - e2.y * t23.y, e2.x * t23.y + e2.y * t23.x);
  o.w = pack_bf16(e3.x * t23.z - e3.y * t23.w, e3.x * t23.w + e3.y * t23.z);
  __stcs(out + idx, o);
}

int launch_rope_apply(const __nv_bfloat16* in, __nv_bfloat16* out, const float2* table, int rows, int heads,
                      cudaStream_t s) {
  const long long total = (long long)rows * heads * (kHeadDim / 8);
  if (total <= 0) return 0;
  const int blocks = (int)((total + 255) / 256);
  const cudaError_t le = launch_kernel(rope_apply_kernel, dim3(blocks), dim3(256), 0, s, 1, reinterpret_cast<const uint4*>(in), reinterpret_cast<uint4*>(out),
                                           table, rows, heads);
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// ------------------------------------------------------------------ positions
// (t, h, w, l) of each token of [text | image | refs]: text i at l = i; image
// token (r, c) of the token grid at (h, w) = (r, c); reference k at the same
// grid coordinates with l = -(k + 1) (blog RoPE table; Chinese summary page).

struct RefDims {
  int n;
  int h[10];
  int w[10];
};

__global__ void positions_kernel(float* __restrict__ pos, int n_txt, int img_h, int img_w, RefDims refs,
                                 int total) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= total) return;
  float t = 0.f, hh = 0.f, ww = 0.f, l = 0.f;
  const int n_img = img_h * img_w;
  if (r < n_txt) {
    l = static_cast<float>(r);
  } else if (r < n_txt + n_img) {
    const int i = r - n_txt;
    hh = static_cast<float>(i / img_w);
    ww = static_cast<float>(i % img_w);
  } else {
    int i = r - n_txt - n_img;
    for (int k = 0; k < refs.n; ++k) {
      const int cnt = refs.h[k] * refs.w[k];
      if (i < cnt) {
        hh = static_cast<float>(i / refs.w[k]);
        ww = static_cast<float>(i % refs.w[k]);
        l = static_cast<float>(-(k + 1));
        break;
      }
      i -= cnt;
    }
  }
  reinterpret_cast<float4*>(pos)[r] = make_float4(t, hh, ww, l);
}

int launch_positions(float* pos, int n_txt, int img_h, int img_w, int n_refs, const int* ref_h, const int* ref_w,
                     cudaStream_t s) {
  RefDims rd{};
  rd.n = n_refs;
  int total = n_txt + img_h * img_w;
  for (int k = 0; k < n_refs && k < 10; ++k) {
    rd.h[k] = ref_h[k];
    rd.w[k] = ref_w[k];
    total += ref_h[k] * ref_w[k];
  }
  if (total <= 0) return 0;
  const cudaError_t le = launch_kernel(positions_kernel, dim3((total + 255) / 256), dim3(256), 0, s, 1, pos, n_txt, img_h, img_w, rd, total);
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// ------------------------------------------------------------------ Euler + CFG
// x <- x + (sigma_next - sigma) * v, v = v_u + g (v_c - v_u) when v_u is given
// (guide "How to Run FLUX 3 Image Klein Locally", "The denoise loop" and
// "Why dropping CFG halves the compute"); optional x0 = x - sigma * v.

__global__ void euler_kernel(float4* __restrict__ x, const float4* __restrict__ vc, const float4* __restrict__ vu,
                             long long n4, float dsigma, float g, float4* __restrict__ x0, float sigma) {
  pdl_trigger();
  pdl_wait();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 v = __ldcs(vc + i);
  if (vu) {
    const float4 u = __ldcs(vu + i);
    v.x = fmaf(g, v.x - u.x, u.x);
    v.y = fmaf(g, v.y - u.y, u.y);
    v.z = fmaf(g, v.z - u.z, u.z);
    v.w = fmaf(g, v.w - u.w, u.w);
  }
  const float4 xv = x[i];
  if (x0) x0[i] = make_float4(fmaf(-sigma, v.x, xv.x), fmaf(-sigma, v.y, xv.y), fmaf(-sigma, v.z, xv.z),
                              fmaf(-sigma, v.w, xv.w));
  x[i] = make_float4(fmaf(dsigma, v.x, xv.x), fmaf(dsigma, v.y, xv.y), fmaf(dsigma, v.z, xv.z),
                     fmaf(dsigma, v.w, xv.w));
}

int launch_euler(float* x, const float* vc, const float* vu, long long n, float dsigma, float g, float* x0,
                 float sigma, cudaStream_t s) {
  if (n <= 0) return 0;
  const long long n4 = n / 4;
  const int blocks = (int)((n4 + 255) / 256);
  const cudaError_t le = launch_kernel(euler_kernel, dim3(blocks), dim3(256), 0, s, 1, reinterpret_cast<float4*>(x), reinterpret_cast<const float4*>(vc),
                                      reinterpret_cast<const float4*>(vu), n4, dsigma, g,
                                      reinterpret_cast<float4*>(x0), sigma);
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

__global__ void to_bf16_kernel(const float4* __restrict__ in, uint2* __restrict__ out, long long n4) {
  pdl_trigger();
  pdl_wait();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = in[i];
  out[i] = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
}

int launch_to_bf16(const float* in, __nv_bfloat16* out, long long n, cudaStream_t s) {
  if (n <= 0) return 0;
  const long long n4 = n / 4;
  const cudaError_t le = launch_kernel(to_bf16_kernel, dim3((int)((n4 + 255) / 256)), dim3(256), 0, s, 1, reinterpret_cast<const float4*>(in),
                                                         reinterpret_cast<uint2*>(out), n4);
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// ------------------------------------------------------------------ GEMV
// y[v][n] = sum_k W[n][k] * f(x[v][k]) (+ add[n]), f = SiLU or identity,
// W bf16 [n_out][k] streamed once for up to 4 vectors. One warp per row.

constexpr int kMaxVec = 4;

__global__ void __launch_bounds__(256) gemv_kernel(const __nv_bfloat16* __restrict__ w, int n_out, int k,
                                                   const float* __restrict__ x, int n_vec, long long x_stride,
                                                   float* __restrict__ y, long long y_stride, int act_silu,
                                                   const float* __restrict__ add) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float xs[];  // [n_vec][k]
  for (int i = threadIdx.x; i < n_vec * k; i += blockDim.x) {
    const int vv = i / k;
    const float e = x[vv * x_stride + (i % k)];
    xs[i] = act_silu ? silu(e) : e;
  }
  __syncthreads();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_out) return;
  const uint4* wr = reinterpret_cast<const uint4*>(w + (long long)row * k);
  float acc[kMaxVec] = {0.f, 0.f, 0.f, 0.f};
  for (int c = lane; c < k / 8; c += 32) {
    const uint4 raw = __ldcs(wr + c);
    const float2 w0 = unpack_bf16(raw.x), w1 = unpack_bf16(raw.y), w2 = unpack_bf16(raw.z), w3 = unpack_bf16(raw.w);
#pragma unroll
    for (int vv = 0; vv < kMaxVec; ++vv) {
      if (vv >= n_vec) break;
      const float* xv = xs + vv * k + 8 * c;
      float a = acc[vv];
      a = fmaf(w0.x, xv[0], a); a = fmaf(w0.y, xv[1], a); a = fmaf(w1.x, xv[2], a); a = fmaf(w1.y, xv[3], a);
      a = fmaf(w2.x, xv[4], a); a = fmaf(w2.y, xv[5], a); a = fmaf(w3.x, xv[6], a); a = fmaf(w3.y, xv[7], a);
      acc[vv] = a;
    }
  }
#pragma unroll
  for (int vv = 0; vv < kMaxVec; ++vv) {
#pragma unroll
    for (int o = 16; o; o >>= 1) acc[vv] += __shfl_xor_sync(0xffffffffu, acc[vv], o);
  }
  if (lane == 0) {
    const float ad = add ? add[row] : 0.f;
    for (int vv = 0; vv < n_vec; ++vv) y[vv * y_stride + row] = acc[vv] + ad;
  }
}

int launch_gemv(const __nv_bfloat16* w, int n_out, int k, const float* x, int n_vec, long long x_stride, float* y,
                long long y_stride, int act_silu, const float* add, cudaStream_t s) {
  if (n_vec < 1 || n_vec > kMaxVec || (k % 8) != 0) return -2;
  const size_t smem = sizeof(float) * n_vec * k;
  static bool configured[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return -1;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxVec * kDim * 4) !=
        cudaSuccess)
      return -1;
    configured[dev] = true;
  }
  const cudaError_t le = launch_kernel(gemv_kernel, dim3((n_out + 7) / 8), dim3(256), smem, s, 1, w, n_out, k, x, n_vec, x_stride, y, y_stride, act_silu, add);
  note_launch();
  return (le == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// ------------------------------------------------------------------ time embedding + modulation
// READING of the pages: the sinusoid of 1000 * sigma is [cos(t f_j), sin(t f_j)]
// with f_j = 10000^(-j/128); the embedder is Linear -> SiLU -> Linear without
// biases (guide "What step distillation removed"); the distilled target-level
// embedder's output is added to every mode's embedding; modulation is
// W * SiLU(e) split into (shift, scale, gate).

__global__ void sinusoid_kernel(float* __restrict__ out, float t0, float t1, float t2) {
  pdl_trigger();
  pdl_wait();
  const int i = threadIdx.x;  // 0..127
  const int v = blockIdx.x;   // 0..2
  const double t = 1000.0 * static_cast<double>(v == 0 ? t0 : (v == 1 ? t1 : t2));
  const double f = pow(10000.0, -static_cast<double>(i) / 128.0);
  double sn, cs;
  sincos(t * f, &sn, &cs);
  out[v * 256 + i] = static_cast<float>(cs);
  out[v * 256 + 128 + i] = static_cast<float>(sn);
}

int launch_time_mod(const TimeModArgs& a, cudaStream_t s) {
  // scratch layout (floats): sin[3][256] | h1[2][3072] | e[2][3072] | tg1[3072] | tg[3072]
  float* sin_v = a.scratch;
  float* h1 = sin_v + 3 * 256;
  float* e = h1 + 2 * kDim;
  float* tg1 = e + 2 * kDim;
  float* tg = tg1 + kDim;
  const cudaError_t le = launch_kernel(sinusoid_kernel, dim3(3), dim3(128), 0, s, 1, sin_v, a.sigma, 0.0f, a.sigma_next);
  note_launch();
  if (le != cudaSuccess || cudaGetLastError() != cudaSuccess) return -1;
  const float* add = nullptr;
  if (a.tt_mlp1) {
    if (launch_gemv(a.tt_mlp1, kDim, 256, sin_v + 2 * 256, 1, 256, tg1, kDim, 0, nullptr, s)) return -1;
    if (launch_gemv(a.tt_mlp2, kDim, kDim, tg1, 1, kDim, tg, kDim, 1, nullptr, s)) return -1;
    add = tg;
  }
  // e[0] = image (sigma), e[1] = context streams (t = 0)
  if (launch_gemv(a.t_mlp1, kDim, 256, sin_v, 2, 256, h1, kDim, 0, nullptr, s)) return -1;
  if (launch_gemv(a.t_mlp2, kDim, kDim, h1, 2, kDim, e, kDim, 1, add, s)) return -1;
  const float* e_img = e;
  const float* e_ctx = e + kDim;
  for (int st = 0; st < 2; ++st) {
    for (int m = 0; m < 3; ++m) {
      if (m == 2 && !a.with_ref) continue;
      const float* ev = (m == 1) ? e_img : e_ctx;
      float* out = a.mod_out + (st * 3 + m) * 3 * kDim;
      if (launch_gemv(a.mod[st][m], 3 * kDim, kDim, ev, 1, kDim, out, 3 * kDim, 1, nullptr, s)) return -1;
    }
  }
  return launch_gemv(a.final_mod, 2 * kDim, kDim, e_img, 1, kDim, a.final_out, 2 * kDim, 1, nullptr, s);
}

// ------------------------------------------------------------------ bounded-wait probe
// Waits on an mbarrier that nothing arrives on, with the given limit, and
// records kErrTimeout. Exercises the same try_wait + %globaltimer bound as
// every pipeline wait, without touching any other kernel.

__global__ void wait_probe_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
      if (mbar_try_wait(&bar, 0)) break;
      if ((i & 63u) == 0u && globaltimer() - t0 > limit_ns) {
        record_error(kErrTimeout, 0x900);
        break;
      }
    }
  }
}

int launch_wait_probe(unsigned long long limit_ns, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(limit_ns);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace klein
