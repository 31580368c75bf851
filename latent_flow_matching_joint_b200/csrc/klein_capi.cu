// C ABI of the Klein denoiser library (declared in include/klein.h): argument
// checking, workspace carving, TMA descriptor set-up and the host-side
// orchestration of block -> stack -> Euler sampler. All arithmetic runs in
// the kernels of gemm.cu, attention.cu and kernels_mem.cu.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <new>

#include "../../include/klein.h"
#include "common.cuh"
#include "internal.h"

namespace klein {

static thread_local char g_msg[512] = "";

static int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

static int cuda_fail(const char* what) {
  const cudaError_t e = cudaGetLastError();
  return fail(KLEIN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Launch counter over all entry points (host threads may launch concurrently).
static std::atomic<long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

int num_sms() {
  static int cached[kMaxDevices] = {0};
  int dev = current_device();
  if (dev < 0) dev = 0;
  if (!cached[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 1;
  }
  return cached[dev];
}

// ------------------------------------------------------------------ launch profiler
// When enabled (klein_profile_begin), CUDA events are recorded on the
// launching stream around each kernel launch of the path, tagged by kernel
// kind; klein_profile_end sums their elapsed times. Off by default: no
// events are recorded then.

// Kinds 0..3 are the four launches of a block over a whole sequence (a joint
// block); a block over a row view of it (a stage-1 block) is recorded as
// kind + kProfStage1 (9..12).
enum ProfKind { kProfModln = 0, kProfGemmIn, kProfAttn, kProfGemmOut, kProfTimeMod, kProfProj, kProfEuler,
                kProfOther, kProfQuant, kProfStage1, kProfKinds = kProfStage1 + 4 };
static_assert(kProfKinds == KLEIN_PROF_KINDS, "profiler kinds and the header's count must agree");

struct Profiler {
  bool on = false;
  int cap = 0;
  int n = 0;
  cudaEvent_t* ev = nullptr;
  int* kind = nullptr;
};
static Profiler g_prof;

static int prof_begin(int kind, cudaStream_t s) {
  if (!g_prof.on || g_prof.n >= g_prof.cap) return -1;
  const int i = g_prof.n++;
  g_prof.kind[i] = kind;
  cudaEventRecord(g_prof.ev[2 * i], s);
  return i;
}

static void prof_end(int i, cudaStream_t s) {
  if (i >= 0) cudaEventRecord(g_prof.ev[2 * i + 1], s);
}

// ------------------------------------------------------------------ TMA maps

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

static int get_encode() {
  if (g_encode) return 0;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return -1;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return 0;
}

int make_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                uint32_t box_inner, uint32_t box_outer, int bytes1) {
  if (get_encode()) return -1;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapDataType dt = bytes1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int make_map_2d_u32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_outer) {
  if (get_encode()) return -1;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int make_map_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                uint64_t s2, uint32_t box0, uint32_t box1, int bytes1) {
  if (get_encode()) return -1;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapDataType dt = bytes1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = g_encode(map, dt, 3, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

// ------------------------------------------------------------------ workspace

static inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
static inline int round_up(int x, int m) { return (x + m - 1) / m * m; }
static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct BlockWs {
  __nv_bfloat16 *h, *q, *k, *vt, *a_out;
  float2* rope;
  float *sa_h, *sa_o;  // FP8 / NVFP4 blocks: per-row scales of the two GEMM inputs
  uint8_t *sf_h, *sf_o;  // NVFP4 blocks: block scales of the two GEMM inputs (atoms over round_up(rows, 256) rows)
  int rows_pad;
  size_t bytes;
};

static BlockWs carve_block(void* base, int batch, int rows) {
  BlockWs w{};
  const int rp = round_up(rows, 128);
  w.rows_pad = rp;
  size_t off = 0;
  auto take = [&](size_t n) -> char* {
    char* p = base ? static_cast<char*>(base) + off : nullptr;
    off += align256(n);
    return p;
  };
  w.h = reinterpret_cast<__nv_bfloat16*>(take((size_t)batch * rows * kDim * 2));
  w.q = reinterpret_cast<__nv_bfloat16*>(take((size_t)batch * kHeads * rp * kHeadDim * 2));
  w.k = reinterpret_cast<__nv_bfloat16*>(take((size_t)batch * kHeads * rp * kHeadDim * 2));
  w.vt = reinterpret_cast<__nv_bfloat16*>(take((size_t)batch * kHeads * rp * kHeadDim * 2));
  w.a_out = reinterpret_cast<__nv_bfloat16*>(take((size_t)batch * rows * kOutK * 2));
  w.rope = reinterpret_cast<float2*>(take((size_t)rows * kPairs * sizeof(float2)));
  w.sa_h = reinterpret_cast<float*>(take((size_t)batch * rows * sizeof(float)));
  w.sa_o = reinterpret_cast<float*>(take((size_t)batch * rows * sizeof(float)));
  const size_t rp256 = (size_t)round_up(rows, 256);
  w.sf_h = reinterpret_cast<uint8_t*>(take((size_t)batch * rp256 * (kDim / 16)));
  w.sf_o = reinterpret_cast<uint8_t*>(take((size_t)batch * rp256 * (kOutK / 16)));
  w.bytes = off;
  return w;
}

// ------------------------------------------------------------------ block

// The block's two big GEMMs run on CTA pairs (256 x 256 tiles) unless the
// library is built with KLEIN_GEMM_PAIR=0 (single CTAs, 128 x 256 tiles).
#ifndef KLEIN_GEMM_PAIR
#define KLEIN_GEMM_PAIR 1
#endif
constexpr int kGemmRowsPerTile = KLEIN_GEMM_PAIR ? 256 : 128;

static int launch_block_gemm(int epi, const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g,
                             cudaStream_t s) {
  return KLEIN_GEMM_PAIR ? launch_gemm_pair(epi, ma, mb, g, s) : launch_gemm(256, epi, ma, mb, g, s);
}

// One block over rows [row0, row0+rows) of x. `rope` holds the view's table
// (row 0 = global row row0). Workspace `w` is carved for (batch, >= rows).
// NVFP4 block (weights with block scales): modLN quantised to NVFP4 ->
// NVFP4 in-projection -> attention -> in-place NVFP4 quantisation of the
// [attention | SwiGLU] rows -> NVFP4 out-projection.
static int block_impl_nvfp4(const klein_block_weights* wt, float* x, int batch, int n_total, int row0, int rows,
                            int n_txt, int n_img, const float2* rope, const float* mod, const BlockWs& w,
                            cudaStream_t s) {
  const int rp = round_up(rows, 128);
  const int kind0 = rows == n_total ? 0 : kProfStage1;
  int pi = prof_begin(kind0 + kProfModln, s);
  if (launch_modln_nvfp4(x, n_total, row0, reinterpret_cast<uint8_t*>(w.h), w.sf_h, w.sa_h, batch, rows, n_txt,
                         n_img, mod, 3 * kDim, s))
    return cuda_fail("modln launch");
  prof_end(pi, s);
  GemmArgs g{};
  g.batch = batch;
  g.rows = rows;
  g.m_tiles_per_b = (rows + 255) / 256;
  g.n_tiles = (kInCols) / 128;
  g.k_blocks = kDim / 256;
  g.q = w.q;
  g.k = w.k;
  g.vt = w.vt;
  g.a_out = w.a_out;
  g.q_norm = wt->q_norm;
  g.k_norm = wt->k_norm;
  g.rope = rope;
  g.rows_pad = rp;
  g.a_scale = w.sa_h;
  g.b_g = wt->w_in_scale;
  pi = prof_begin(kind0 + kProfGemmIn, s);
  int rc = launch_gemm_nvfp4(kEpiQKV, w.h, kDim / 2, w.sf_h, wt->w_in, wt->w_in_sf, g, kInCols, s);
  if (rc == -2) return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  if (rc) return cuda_fail("in-projection GEMM launch");
  prof_end(pi, s);
  AttnArgs at{};
  at.batch = batch;
  at.heads = kHeads;
  at.rows = rows;
  at.rows_pad = rp;
  at.q = w.q;
  at.k = w.k;
  at.vt = w.vt;
  at.out = w.a_out;
  at.out_ld = kOutK;
  at.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(128.0));
  pi = prof_begin(kind0 + kProfAttn, s);
  if (launch_attention(at, s)) return cuda_fail("attention launch");
  prof_end(pi, s);
  pi = prof_begin(kProfQuant, s);
  if (launch_quantize_nvfp4(w.a_out, kOutK, 0, reinterpret_cast<uint8_t*>(w.a_out), (long long)kOutK * 2, w.sf_o,
                            w.sa_o, nullptr, batch, rows, round_up(rows, 256), kOutK, s))
    return cuda_fail("quantisation launch");
  prof_end(pi, s);
  GemmArgs o{};
  o.batch = batch;
  o.rows = rows;
  o.m_tiles_per_b = (rows + 255) / 256;
  o.n_tiles = kDim / 128;
  o.k_blocks = kOutK / 256;
  o.n_fastest = 1;
  o.x = x;
  o.x_bstride = n_total;
  o.x_row0 = row0;
  o.mod = mod;
  o.n_txt = n_txt;
  o.n_img = n_img;
  o.a_scale = w.sa_o;
  o.b_g = wt->w_out_scale;
  pi = prof_begin(kind0 + kProfGemmOut, s);
  // the codes sit at the start of each bf16 [attention | SwiGLU] row (pitch 24576 bytes)
  rc = launch_gemm_nvfp4(kEpiResid, w.a_out, (long long)kOutK * 2, w.sf_o, wt->w_out, wt->w_out_sf, o, kDim, s);
  if (rc == -2) return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  if (rc == -3) return fail(KLEIN_ERR_SHAPE, "the out-projection's N must be a multiple of 256");
  if (rc) return cuda_fail("out-projection GEMM launch");
  prof_end(pi, s);
  return KLEIN_OK;
}

static int block_impl(const klein_block_weights* wt, float* x, int batch, int n_total, int row0, int rows,
                      int n_txt, int n_img, const float2* rope, const float* mod, const BlockWs& w,
                      cudaStream_t s) {
  if (wt->w_in_sf) return block_impl_nvfp4(wt, x, batch, n_total, row0, rows, n_txt, n_img, rope, mod, w, s);
  const int rp = round_up(rows, 128);
  // Rowwise FP8 blocks: both GEMMs on e4m3 codes (CTA pairs); the GEMM
  // inputs are quantised per row where they are made (modLN) or just before
  // the out-projection (in place, over the bf16 [attention | SwiGLU] rows).
  const bool f8 = wt->w_in_scale != nullptr;
  const int rows_per_tile = f8 ? 256 : kGemmRowsPerTile;
  const int kind0 = rows == n_total ? 0 : kProfStage1;  // profiler: joint block, or a row view
  // a4: modulated LayerNorm
  int pi = prof_begin(kind0 + kProfModln, s);
  const int mrc = f8 ? launch_modln_e4m3(x, n_total, row0, reinterpret_cast<uint8_t*>(w.h), w.sa_h, batch, rows,
                                         n_txt, n_img, mod, 3 * kDim, s)
                     : launch_modln(x, n_total, row0, w.h, batch, rows, n_txt, n_img, mod, 3 * kDim, 0, s);
  if (mrc) return cuda_fail("modln launch");
  prof_end(pi, s);
  // a5: fused in-projection
  CUtensorMap m_h, m_win, m_aout, m_wout;
  const int eb = f8 ? 1 : 2;                // operand bytes per element
  const uint32_t bk = f8 ? 128 : 64;        // elements per 128-byte K box
  if (make_map_3d(&m_h, w.h, kDim, rows, batch, (uint64_t)kDim * eb, (uint64_t)rows * kDim * eb, bk, 128, f8) ||
      make_map_2d(&m_win, wt->w_in, kDim, kInCols, (uint64_t)kDim * eb, bk, 128, f8) ||
      // the out-projection's A keeps the bf16 row pitch: FP8 codes are written in place
      make_map_3d(&m_aout, w.a_out, kOutK, rows, batch, (uint64_t)kOutK * 2, (uint64_t)rows * kOutK * 2, bk, 128,
                  f8) ||
      make_map_2d(&m_wout, wt->w_out, kOutK, kDim, (uint64_t)kOutK * eb, bk, 128, f8))
    return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  GemmArgs g{};
  g.batch = batch;
  g.rows = rows;
  g.m_tiles_per_b = (rows + rows_per_tile - 1) / rows_per_tile;
  g.n_tiles = 36 + kMlp / 128;
  g.k_blocks = kDim / static_cast<int>(bk);
  g.b_split = 36;
  g.q = w.q;
  g.k = w.k;
  g.vt = w.vt;
  g.a_out = w.a_out;
  g.q_norm = wt->q_norm;
  g.k_norm = wt->k_norm;
  g.rope = rope;
  g.rows_pad = rp;
  g.a_scale = w.sa_h;
  g.b_scale = wt->w_in_scale;
  pi = prof_begin(kind0 + kProfGemmIn, s);
  if (f8 ? launch_gemm_pair(kEpiQKV, m_h, m_win, g, s, 1) : launch_block_gemm(kEpiQKV, m_h, m_win, g, s))
    return cuda_fail("in-projection GEMM launch");
  prof_end(pi, s);
  // a6: attention
  AttnArgs at{};
  at.batch = batch;
  at.heads = kHeads;
  at.rows = rows;
  at.rows_pad = rp;
  at.q = w.q;
  at.k = w.k;
  at.vt = w.vt;
  at.out = w.a_out;
  at.out_ld = kOutK;
  at.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(128.0));
  pi = prof_begin(kind0 + kProfAttn, s);
  if (launch_attention(at, s)) return cuda_fail("attention launch");
  prof_end(pi, s);
  if (f8) {
    pi = prof_begin(kProfQuant, s);
    if (launch_quantize_rows(w.a_out, kOutK, reinterpret_cast<uint8_t*>(w.a_out), (long long)kOutK * 2, w.sa_o,
                             (long long)batch * rows, kOutK, s))
      return cuda_fail("quantisation launch");
    prof_end(pi, s);
  }
  // a7: out-projection + gated residual
  GemmArgs o{};
  o.batch = batch;
  o.rows = rows;
  o.m_tiles_per_b = (rows + rows_per_tile - 1) / rows_per_tile;
  o.n_tiles = kDim / 256;
  o.k_blocks = kOutK / static_cast<int>(bk);
  o.n_fastest = 1;
  o.x = x;
  o.x_bstride = n_total;
  o.x_row0 = row0;
  o.mod = mod;
  o.n_txt = n_txt;
  o.n_img = n_img;
  o.a_scale = w.sa_o;
  o.b_scale = wt->w_out_scale;
  pi = prof_begin(kind0 + kProfGemmOut, s);
  if (f8 ? launch_gemm_pair(kEpiResid, m_aout, m_wout, o, s, 1) : launch_block_gemm(kEpiResid, m_aout, m_wout, o, s))
    return cuda_fail("out-projection GEMM launch");
  prof_end(pi, s);
  return KLEIN_OK;
}

static int check_seq(const klein_seq* q, int* n_img, int* n_ref, int* n_total) {
  if (!q) return fail(KLEIN_ERR_INVALID_ARG, "seq is NULL");
  if (q->batch < 1 || q->batch > 64) return fail(KLEIN_ERR_SHAPE, "batch %d out of range", q->batch);
  if (q->n_txt < 1) return fail(KLEIN_ERR_SHAPE, "n_txt must be >= 1");
  if (q->img_h < 1 || q->img_w < 1) return fail(KLEIN_ERR_SHAPE, "image grid must be >= 1x1");
  if (q->n_refs < 0 || q->n_refs > KLEIN_MAX_REFS) return fail(KLEIN_ERR_SHAPE, "n_refs out of range");
  long long ni = (long long)q->img_h * q->img_w, nr = 0;
  for (int k = 0; k < q->n_refs; ++k) {
    if (q->ref_h[k] < 1 || q->ref_w[k] < 1) return fail(KLEIN_ERR_SHAPE, "reference %d grid must be >= 1x1", k);
    nr += (long long)q->ref_h[k] * q->ref_w[k];
  }
  const long long nt = q->n_txt + ni + nr;
  if (nt > (1 << 20)) return fail(KLEIN_ERR_SHAPE, "sequence too long");
  if (n_img) *n_img = static_cast<int>(ni);
  if (n_ref) *n_ref = static_cast<int>(nr);
  if (n_total) *n_total = static_cast<int>(nt);
  return KLEIN_OK;
}

// ------------------------------------------------------------------ stack

struct StackWs {
  float* x;           // residual stream [batch][n_total][3072]
  float* pos;
  float2* rope;
  float* mod;        // [2][3][3][3072]
  float* fmod;       // [2][3072]
  float* tscratch;   // 8 * 3072 floats
  __nv_bfloat16* lat_bf;  // [max(n_img, n_ref)][128]
  float* v;          // [batch][n_img][128]
  float* txt;        // [batch][n_txt][3072] projected text (models with txt_in)
  float* s1_txt;     // [batch][n_txt][3072] stage-1 output of the text stream (base model cache)
  float* s1_ref;     // [n_ref][3072] stage-1 output of the reference stream (base model cache)
  BlockWs blk;
  size_t bytes;
};

static StackWs carve_stack(void* base, int batch, int n_total, int n_img, int n_ref) {
  StackWs w{};
  size_t off = 0;
  auto take = [&](size_t n) -> char* {
    char* p = base ? static_cast<char*>(base) + off : nullptr;
    off += align256(n);
    return p;
  };
  w.x = reinterpret_cast<float*>(take((size_t)batch * n_total * kDim * sizeof(float)));
  w.pos = reinterpret_cast<float*>(take((size_t)n_total * 4 * sizeof(float)));
  w.rope = reinterpret_cast<float2*>(take((size_t)n_total * kPairs * sizeof(float2)));
  w.mod = reinterpret_cast<float*>(take((size_t)2 * 3 * 3 * kDim * sizeof(float)));
  w.fmod = reinterpret_cast<float*>(take((size_t)2 * kDim * sizeof(float)));
  w.tscratch = reinterpret_cast<float*>(take((size_t)8 * kDim * sizeof(float)));
  w.lat_bf = reinterpret_cast<__nv_bfloat16*>(take((size_t)(n_img > n_ref ? n_img : n_ref) * kLatent * 2));
  w.v = reinterpret_cast<float*>(take((size_t)batch * n_img * kLatent * sizeof(float)));
  w.txt = reinterpret_cast<float*>(take((size_t)batch * (n_total - n_img - n_ref) * kDim * sizeof(float)));
  w.s1_txt = reinterpret_cast<float*>(take((size_t)batch * (n_total - n_img - n_ref) * kDim * sizeof(float)));
  w.s1_ref = reinterpret_cast<float*>(take((size_t)n_ref * kDim * sizeof(float)));
  w.blk = carve_block(base ? static_cast<char*>(base) + off : nullptr, batch, n_total);
  off += w.blk.bytes;
  w.bytes = off;
  return w;
}

}  // namespace klein

using namespace klein;

struct klein_model {
  klein_model_desc d;
};

extern "C" {

const char* klein_last_error(void) { return g_msg; }

int klein_version(void) { return 103; }

long long klein_launch_count(void) { return g_launches; }

// Reads and clears the device error word that bounded waits write.
static int take_device_error(unsigned* site) {
  unsigned err = 0, where = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&err, g_klein_error, sizeof(err)) != cudaSuccess ||
      cudaMemcpyFromSymbol(&where, g_klein_error_site, sizeof(where)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_klein_error, &zero, sizeof(zero)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_klein_error_site, &zero, sizeof(zero)) != cudaSuccess)
    return cuda_fail("reading the device error word");
  if (site) *site = where;
  if (err & kErrTimeout) return fail(KLEIN_ERR_TIMEOUT, "device wait gave up at site 0x%x", where);
  if (err) return fail(KLEIN_ERR_CUDA, "device error bits 0x%x at site 0x%x", err, where);
  g_msg[0] = 0;
  return KLEIN_OK;
}

int klein_device_status(unsigned* site) {
  if (cudaDeviceSynchronize() != cudaSuccess) return cuda_fail("cudaDeviceSynchronize");
  return take_device_error(site);
}

int klein_sync(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return cuda_fail("cudaStreamSynchronize");
  return take_device_error(nullptr);
}

int klein_set_wait_limit_ns(unsigned long long ns) {
  if (ns == 0) return fail(KLEIN_ERR_INVALID_ARG, "wait limit must be > 0");
  if (cudaMemcpyToSymbol(g_klein_wait_limit_ns, &ns, sizeof(ns)) != cudaSuccess)
    return cuda_fail("setting the wait limit");
  return KLEIN_OK;
}

int klein_wait_probe(unsigned long long limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return fail(KLEIN_ERR_INVALID_ARG, "probe limit out of range");
  if (launch_wait_probe(limit_ns, static_cast<cudaStream_t>(stream))) return cuda_fail("probe launch");
  return KLEIN_OK;
}

int klein_profile_begin(int max_launches) {
  if (g_prof.on) return fail(KLEIN_ERR_INVALID_ARG, "profiler already running");
  if (max_launches < 1 || max_launches > (1 << 20)) return fail(KLEIN_ERR_INVALID_ARG, "max_launches out of range");
  g_prof.ev = new (std::nothrow) cudaEvent_t[2 * (size_t)max_launches];
  g_prof.kind = new (std::nothrow) int[max_launches];
  if (!g_prof.ev || !g_prof.kind) {
    delete[] g_prof.ev;
    delete[] g_prof.kind;
    g_prof.ev = nullptr;
    g_prof.kind = nullptr;
    return fail(KLEIN_ERR_INVALID_ARG, "out of host memory");
  }
  for (int i = 0; i < 2 * max_launches; ++i) {
    if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(g_prof.ev[j]);
      delete[] g_prof.ev;
      delete[] g_prof.kind;
      g_prof.ev = nullptr;
      g_prof.kind = nullptr;
      return cuda_fail("cudaEventCreate");
    }
  }
  g_prof.cap = max_launches;
  g_prof.n = 0;
  g_prof.on = true;
  return KLEIN_OK;
}

int klein_profile_end(double* ms, int* launches) {
  if (!g_prof.on) return fail(KLEIN_ERR_INVALID_ARG, "profiler not running");
  g_prof.on = false;
  int rc = KLEIN_OK;
  for (int k = 0; k < kProfKinds; ++k) {
    if (ms) ms[k] = 0.0;
    if (launches) launches[k] = 0;
  }
  if (g_prof.n > 0 && cudaEventSynchronize(g_prof.ev[2 * g_prof.n - 1]) != cudaSuccess) rc = cuda_fail("event sync");
  for (int i = 0; rc == KLEIN_OK && i < g_prof.n; ++i) {
    float t = 0.f;
    if (cudaEventElapsedTime(&t, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess) {
      rc = cuda_fail("cudaEventElapsedTime");
      break;
    }
    if (ms) ms[g_prof.kind[i]] += t;
    if (launches) launches[g_prof.kind[i]] += 1;
  }
  const int dropped = g_prof.n >= g_prof.cap;
  for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
  delete[] g_prof.ev;
  delete[] g_prof.kind;
  g_prof.ev = nullptr;
  g_prof.kind = nullptr;
  g_prof.cap = g_prof.n = 0;
  if (rc == KLEIN_OK && dropped) return fail(KLEIN_ERR_WORKSPACE, "profiler capacity reached; later launches not timed");
  return rc;
}

int klein_seq_tokens(const klein_seq* seq, int* n_img, int* n_ref, int* n_total) {
  return check_seq(seq, n_img, n_ref, n_total);
}

int klein_pad_text_len(int n) {
  if (n < 0) return -1;
  return (n + 79) / 80 * 80;
}

int klein_sigma_schedule(int steps, float shift, float* sigmas) {
  if (steps < 1 || !sigmas) return fail(KLEIN_ERR_INVALID_ARG, "steps must be >= 1 and sigmas non-NULL");
  if (!(shift > 0.f)) return fail(KLEIN_ERR_INVALID_ARG, "shift must be > 0");
  const double s = shift;
  for (int i = 0; i < steps; ++i) {
    // evenly spaced from 1 down to 1/steps
    const double base = steps == 1 ? 1.0 : 1.0 + (1.0 / steps - 1.0) * i / (steps - 1);
    sigmas[i] = static_cast<float>(s * base / (1.0 + (s - 1.0) * base));
  }
  sigmas[steps] = 0.f;
  return KLEIN_OK;
}

int klein_positions(const klein_seq* seq, float* pos, void* stream) {
  int rc = check_seq(seq, nullptr, nullptr, nullptr);
  if (rc) return rc;
  if (!pos || !aligned16(pos)) return fail(KLEIN_ERR_ALIGN, "pos must be a 16-byte aligned device pointer");
  if (launch_positions(pos, seq->n_txt, seq->img_h, seq->img_w, seq->n_refs, seq->ref_h, seq->ref_w,
                       static_cast<cudaStream_t>(stream)))
    return cuda_fail("positions launch");
  return KLEIN_OK;
}

size_t klein_block_workspace_size(int batch, int rows) {
  if (batch < 1 || rows < 1) return 0;
  return carve_block(nullptr, batch, rows).bytes;
}

static int check_block_weights(const klein_block_weights* w) {
  if (!w || !w->w_in || !w->w_out || !w->q_norm || !w->k_norm)
    return fail(KLEIN_ERR_INVALID_ARG, "block weights incomplete");
  if (!aligned16(w->w_in) || !aligned16(w->w_out) || !aligned16(w->q_norm) || !aligned16(w->k_norm))
    return fail(KLEIN_ERR_ALIGN, "block weights must be 16-byte aligned");
  if ((w->w_in_scale == nullptr) != (w->w_out_scale == nullptr))
    return fail(KLEIN_ERR_INVALID_ARG, "FP8 block weights need both w_in_scale and w_out_scale");
  if ((w->w_in_sf == nullptr) != (w->w_out_sf == nullptr))
    return fail(KLEIN_ERR_INVALID_ARG, "NVFP4 block weights need both w_in_sf and w_out_sf");
  if (w->w_in_sf && !w->w_in_scale)
    return fail(KLEIN_ERR_INVALID_ARG, "NVFP4 block weights need their second-level scales (w_in_scale, w_out_scale)");
  if ((w->w_in_scale && !aligned16(w->w_in_scale)) || (w->w_out_scale && !aligned16(w->w_out_scale)) ||
      (w->w_in_sf && !aligned16(w->w_in_sf)) || (w->w_out_sf && !aligned16(w->w_out_sf)))
    return fail(KLEIN_ERR_ALIGN, "weight scales must be 16-byte aligned");
  return KLEIN_OK;
}

// Shapes of a block call: a non-empty row range inside [0, n_total) and
// stream sizes that fit the sequence (text rows, then image rows, the rest
// references).
static int check_block_rows(int batch, int n_total, int row0, int rows, int n_txt, int n_img) {
  if (batch < 1 || n_total < 1 || rows < 1 || row0 < 0 || (long long)row0 + rows > n_total)
    return fail(KLEIN_ERR_SHAPE, "row range [%d, %lld) outside [0, %d)", row0, (long long)row0 + rows, n_total);
  if (n_txt < 0 || n_img < 0) return fail(KLEIN_ERR_SHAPE, "negative stream sizes");
  if ((long long)n_txt + n_img > n_total)
    return fail(KLEIN_ERR_SHAPE, "n_txt + n_img = %lld exceeds n_total = %d", (long long)n_txt + n_img, n_total);
  return KLEIN_OK;
}

int klein_block_forward(const klein_block_weights* w, void* x, int batch, int n_total, int row0, int rows,
                        int n_txt, int n_img, const float* pos, const float* mod, void* ws, size_t ws_bytes,
                        void* stream) {
  int rc = check_block_weights(w);
  if (rc) return rc;
  if (!x || !pos || !mod || !ws) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(x) || !aligned16(pos) || !aligned16(mod) || !aligned16(ws))
    return fail(KLEIN_ERR_ALIGN, "pointers must be 16-byte aligned");
  if ((rc = check_block_rows(batch, n_total, row0, rows, n_txt, n_img))) return rc;
  const BlockWs bw = carve_block(ws, batch, rows);
  if (ws_bytes < bw.bytes) return fail(KLEIN_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, bw.bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_rope_table(pos + (size_t)row0 * 4, bw.rope, rows, 10000.f, s)) return cuda_fail("rope table");
  return block_impl(w, static_cast<float*>(x), batch, n_total, row0, rows, n_txt, n_img, bw.rope, mod, bw,
                    s);
}

int klein_model_create(klein_model** out, const klein_model_desc* d) {
  if (!out || !d) return fail(KLEIN_ERR_INVALID_ARG, "NULL argument");
  *out = nullptr;
  if (d->n_stage1 < 0 || d->n_joint < 0) return fail(KLEIN_ERR_SHAPE, "negative block counts");
  for (int m = 0; m < 3; ++m) {
    if (d->n_stage1 > 0 && !d->stage1[m] && m != 2) return fail(KLEIN_ERR_INVALID_ARG, "stage-1 weights missing");
    for (int i = 0; d->stage1[m] && i < d->n_stage1; ++i) {
      int rc = check_block_weights(&d->stage1[m][i]);
      if (rc) return rc;
    }
  }
  if (d->n_joint > 0 && !d->joint) return fail(KLEIN_ERR_INVALID_ARG, "joint weights missing");
  for (int i = 0; i < d->n_joint; ++i) {
    int rc = check_block_weights(&d->joint[i]);
    if (rc) return rc;
  }
  if (!d->img_in || !d->t_mlp1 || !d->t_mlp2 || !d->final_mod || !d->final_out)
    return fail(KLEIN_ERR_INVALID_ARG, "model weights incomplete");
  for (int st = 0; st < 2; ++st)
    for (int m = 0; m < 2; ++m)
      if (!d->mod[st][m]) return fail(KLEIN_ERR_INVALID_ARG, "modulation weights incomplete");
  if ((d->tt_mlp1 == nullptr) != (d->tt_mlp2 == nullptr))
    return fail(KLEIN_ERR_INVALID_ARG, "target embedder needs both layers");
  if (d->txt_in && !aligned16(d->txt_in)) return fail(KLEIN_ERR_ALIGN, "txt_in must be 16-byte aligned");
  klein_model* m = new (std::nothrow) klein_model;
  if (!m) return fail(KLEIN_ERR_INVALID_ARG, "out of host memory");
  m->d = *d;
  *out = m;
  return KLEIN_OK;
}

void klein_model_destroy(klein_model* m) { delete m; }

size_t klein_stack_workspace_size(const klein_seq* seq) {
  int ni = 0, nr = 0, nt = 0;
  if (check_seq(seq, &ni, &nr, &nt)) return 0;
  return carve_stack(nullptr, seq->batch, nt, ni, nr).bytes;
}

int klein_op_time_mod(const klein_model* m, float sigma, float sigma_next, int with_ref, float* mod_out,
                      float* final_out, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !mod_out || !final_out || !ws) return fail(KLEIN_ERR_INVALID_ARG, "NULL argument");
  if (ws_bytes < 8 * kDim * sizeof(float)) return fail(KLEIN_ERR_WORKSPACE, "time-mod workspace too small");
  if (with_ref && (!m->d.mod[0][2] || !m->d.mod[1][2]))
    return fail(KLEIN_ERR_INVALID_ARG, "reference modulation weights missing");
  TimeModArgs a{};
  a.t_mlp1 = static_cast<const __nv_bfloat16*>(m->d.t_mlp1);
  a.t_mlp2 = static_cast<const __nv_bfloat16*>(m->d.t_mlp2);
  a.tt_mlp1 = static_cast<const __nv_bfloat16*>(m->d.tt_mlp1);
  a.tt_mlp2 = static_cast<const __nv_bfloat16*>(m->d.tt_mlp2);
  for (int st = 0; st < 2; ++st)
    for (int md = 0; md < 3; ++md) a.mod[st][md] = static_cast<const __nv_bfloat16*>(m->d.mod[st][md]);
  a.final_mod = static_cast<const __nv_bfloat16*>(m->d.final_mod);
  a.sigma = sigma;
  a.sigma_next = sigma_next;
  a.with_ref = with_ref;
  a.scratch = static_cast<float*>(ws);
  a.mod_out = mod_out;
  a.final_out = final_out;
  if (launch_time_mod(a, static_cast<cudaStream_t>(stream))) return cuda_fail("time/modulation launch");
  return KLEIN_OK;
}

constexpr int kTextStack = 8 * 2560;  // eight 2560-wide encoder layers per text token

// Text input projection (models with txt_in): w.txt = text [B][n_txt][20480] x txt_in^T.
static int project_text(const klein_model* m, const void* text, const klein_seq* seq, const StackWs& w,
                        cudaStream_t s) {
  const int B = seq->batch;
  const int n_txt = seq->n_txt;
  CUtensorMap ma, mb;
  if (make_map_3d(&ma, text, kTextStack, n_txt, B, (uint64_t)kTextStack * 2, (uint64_t)n_txt * kTextStack * 2, 64,
                  128) ||
      make_map_2d(&mb, m->d.txt_in, kTextStack, kDim, (uint64_t)kTextStack * 2, 64, 128))
    return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  GemmArgs g{};
  g.batch = B;
  g.rows = n_txt;
  g.m_tiles_per_b = (n_txt + kGemmRowsPerTile - 1) / kGemmRowsPerTile;
  g.n_tiles = kDim / 256;
  g.k_blocks = kTextStack / 64;
  g.out = w.txt;
  g.out_ld = kDim;
  g.out_bstride = n_txt;
  const int pi = prof_begin(kProfProj, s);
  if (launch_block_gemm(kEpiF32, ma, mb, g, s)) return cuda_fail("text projection launch");
  prof_end(pi, s);
  return KLEIN_OK;
}

// Stage-1 cache of the text and reference streams. Their stage-1 output does
// not depend on the noise level when the model has no target-level embedder
// (base model: those streams are always modulated at t = 0), so a denoise
// computes it at the first step and reuses it afterwards.
enum StageOneCache { kCacheNone = 0, kCacheStore = 1, kCacheLoad = 2 };

static int copy_rows_f32(float* dst, const float* src, size_t rows, cudaStream_t s) {
  return cudaMemcpyAsync(dst, src, rows * kDim * sizeof(float), cudaMemcpyDeviceToDevice, s) == cudaSuccess
             ? KLEIN_OK
             : cuda_fail("stage-1 cache copy");
}

static int stack_impl(const klein_model* m, const float* latents, const void* text, const float* refs,
                      float sigma, float sigma_next, const klein_seq* seq, float* v_out, const StackWs& w,
                      int n_img, int n_ref, int n_total, bool prepared, int cache, cudaStream_t s) {
  const klein_model_desc& d = m->d;
  const int B = seq->batch;
  const int n_txt = seq->n_txt;
  const bool load = cache == kCacheLoad;
  int rc;
  if (!prepared) {
    if (launch_positions(w.pos, n_txt, seq->img_h, seq->img_w, seq->n_refs, seq->ref_h, seq->ref_w, s) ||
        launch_rope_table(w.pos, w.rope, n_total, 10000.f, s))
      return cuda_fail("positions / rope table");
    if (d.txt_in && (rc = project_text(m, text, seq, w, s))) return rc;
  }
  // a2: timestep embedding + modulation
  int pi = prof_begin(kProfTimeMod, s);
  rc = klein_op_time_mod(m, sigma, sigma_next, n_ref > 0, w.mod, w.fmod, w.tscratch, 8 * kDim * sizeof(float), s);
  if (rc) return rc;
  prof_end(pi, s);
  // a3: assemble [text | image | reference] rows of x
  pi = prof_begin(kProfOther, s);
  if (load) {
    for (int b = 0; b < B; ++b)
      if ((rc = copy_rows_f32(w.x + (size_t)b * n_total * kDim, w.s1_txt + (size_t)b * n_txt * kDim, n_txt, s)))
        return rc;
    if (n_ref && (rc = copy_rows_f32(w.x + (size_t)(n_txt + n_img) * kDim, w.s1_ref, n_ref, s))) return rc;
  } else if (d.txt_in) {
    for (int b = 0; b < B; ++b)
      if (cudaMemcpyAsync(w.x + (size_t)b * n_total * kDim, w.txt + (size_t)b * n_txt * kDim,
                          (size_t)n_txt * kDim * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return cuda_fail("text rows");
  } else if (launch_rows_to_f32(static_cast<const __nv_bfloat16*>(text), n_txt, w.x, n_total, 0, B, n_txt, s)) {
    return cuda_fail("text rows");
  }
  prof_end(pi, s);
  auto project = [&](const float* lat, int rows, const void* wproj, int row0) -> int {
    const int pc = prof_begin(kProfProj, s);
    if (launch_to_bf16(lat, w.lat_bf, (long long)rows * kLatent, s)) return cuda_fail("latent cast");
    prof_end(pc, s);
    CUtensorMap ma, mb;
    if (make_map_3d(&ma, w.lat_bf, kLatent, rows, 1, kLatent * 2, (uint64_t)rows * kLatent * 2, 64, 128) ||
        make_map_2d(&mb, wproj, kLatent, kDim, kLatent * 2, 64, 128))
      return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    GemmArgs g{};
    g.batch = 1;
    g.rows = rows;
    g.m_tiles_per_b = (rows + 127) / 128;
    g.n_tiles = kDim / 256;
    g.k_blocks = kLatent / 64;
    g.out = w.x;
    g.out_ld = kDim;
    g.out_bstride = n_total;
    g.out_row0 = row0;
    g.replicate = B;
    const int pj = prof_begin(kProfProj, s);
    if (launch_gemm(256, kEpiF32, ma, mb, g, s)) return cuda_fail("input projection launch");
    prof_end(pj, s);
    return KLEIN_OK;
  };
  if ((rc = project(latents, n_img, d.img_in, n_txt))) return rc;
  if (n_ref && !load && (rc = project(refs, n_ref, d.ref_in, n_txt + n_img))) return rc;
  // a8 stage 1: each stream through its own blocks, attending to itself.
  // The image and reference streams start from the same latents in every
  // batch item (the batch only varies the text, e.g. guidance's cond and
  // uncond prompts) and stage 1 never mixes streams, so they are computed
  // for batch item 0 and copied to the others.
  const int lo[3] = {0, n_txt, n_txt + n_img};
  const int cnt[3] = {n_txt, n_img, n_ref};
  for (int md = 0; md < 3; ++md) {
    if (cnt[md] == 0 || (load && md != 1)) continue;
    const int nb = md == 0 ? B : 1;
    for (int i = 0; i < d.n_stage1; ++i) {
      rc = block_impl(&d.stage1[md][i], w.x, nb, n_total, lo[md], cnt[md], n_txt, n_img,
                      w.rope + (size_t)lo[md] * kPairs, w.mod, w.blk, s);
      if (rc) return rc;
    }
  }
  if (cache == kCacheStore) {
    for (int b = 0; b < B; ++b)
      if ((rc = copy_rows_f32(w.s1_txt + (size_t)b * n_txt * kDim, w.x + (size_t)b * n_total * kDim, n_txt, s)))
        return rc;
    if (n_ref && (rc = copy_rows_f32(w.s1_ref, w.x + (size_t)(n_txt + n_img) * kDim, n_ref, s))) return rc;
  }
  if (d.n_stage1 > 0) {
    for (int b = 1; b < B; ++b) {
      if (cudaMemcpyAsync(w.x + ((size_t)b * n_total + n_txt) * kDim, w.x + (size_t)n_txt * kDim,
                          (size_t)(n_img + n_ref) * kDim * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return cuda_fail("stage-1 stream copy");
    }
  }
  // a8 stage 2: joint blocks over everything
  for (int i = 0; i < d.n_joint; ++i) {
    rc = block_impl(&d.joint[i], w.x, B, n_total, 0, n_total, n_txt, n_img, w.rope, w.mod + 9 * kDim, w.blk, s);
    if (rc) return rc;
  }
  // a9: output layer on image rows
  pi = prof_begin(kProfModln, s);
  if (launch_modln(w.x, n_total, n_txt, w.blk.h, B, n_img, n_txt, n_img, w.fmod, 0, 1, s))
    return cuda_fail("final modln");
  prof_end(pi, s);
  CUtensorMap ma, mb;
  if (make_map_3d(&ma, w.blk.h, kDim, n_img, B, kDim * 2, (uint64_t)n_img * kDim * 2, 64, 128) ||
      make_map_2d(&mb, d.final_out, kDim, kLatent, kDim * 2, 64, 128))
    return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  GemmArgs g{};
  g.batch = B;
  g.rows = n_img;
  g.m_tiles_per_b = (n_img + 127) / 128;
  g.n_tiles = 1;
  g.k_blocks = kDim / 64;
  g.out = v_out;
  g.out_ld = kLatent;
  g.out_bstride = n_img;
  g.out_row0 = 0;
  pi = prof_begin(kProfProj, s);
  if (launch_gemm(128, kEpiF32, ma, mb, g, s)) return cuda_fail("output projection launch");
  prof_end(pi, s);
  return KLEIN_OK;
}

static int check_stack_args(const klein_model* m, const void* latents, const void* text, const float* refs,
                            const klein_seq* seq, void* ws, size_t ws_bytes, int* ni, int* nr, int* nt) {
  if (!m) return fail(KLEIN_ERR_INVALID_ARG, "model is NULL");
  int rc = check_seq(seq, ni, nr, nt);
  if (rc) return rc;
  if (!latents || !text || !ws) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(latents) || !aligned16(text) || !aligned16(ws) || (refs && !aligned16(refs)))
    return fail(KLEIN_ERR_ALIGN, "pointers must be 16-byte aligned");
  if (*nr > 0 && (!refs || !m->d.ref_in || !m->d.mod[0][2] || !m->d.mod[1][2] ||
                  (m->d.n_stage1 > 0 && !m->d.stage1[2])))
    return fail(KLEIN_ERR_INVALID_ARG, "references given but reference weights or latents missing");
  const size_t need = carve_stack(nullptr, seq->batch, *nt, *ni, *nr).bytes;
  if (ws_bytes < need) return fail(KLEIN_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  return KLEIN_OK;
}

int klein_stack_forward(const klein_model* m, const float* latents, const void* text, const float* refs,
                        float sigma, float sigma_next, const klein_seq* seq, float* v_out, void* ws,
                        size_t ws_bytes, void* stream) {
  int ni = 0, nr = 0, nt = 0;
  int rc = check_stack_args(m, latents, text, refs, seq, ws, ws_bytes, &ni, &nr, &nt);
  if (rc) return rc;
  if (!v_out || !aligned16(v_out)) return fail(KLEIN_ERR_ALIGN, "v_out must be a 16-byte aligned device pointer");
  const StackWs w = carve_stack(ws, seq->batch, nt, ni, nr);
  return stack_impl(m, latents, text, refs, sigma, sigma_next, seq, v_out, w, ni, nr, nt, false, kCacheNone,
                    static_cast<cudaStream_t>(stream));
}

int klein_denoise(const klein_model* m, float* latents, const void* text, const float* refs, int steps, float cfg,
                  float shift, const klein_seq* seq, float* x0_out, int x0_every_step, void* ws, size_t ws_bytes,
                  void* stream) {
  int ni = 0, nr = 0, nt = 0;
  int rc = check_stack_args(m, latents, text, refs, seq, ws, ws_bytes, &ni, &nr, &nt);
  if (rc) return rc;
  if (steps < 1 || steps > 1000) return fail(KLEIN_ERR_INVALID_ARG, "steps out of range");
  const bool guided = cfg > 1.0f;
  if (guided && seq->batch != 2) return fail(KLEIN_ERR_SHAPE, "guidance needs batch 2 (cond, uncond)");
  if (!guided && seq->batch != 1) return fail(KLEIN_ERR_SHAPE, "unguided sampling needs batch 1");
  if (x0_out && !aligned16(x0_out)) return fail(KLEIN_ERR_ALIGN, "x0_out must be 16-byte aligned");
  float* sig = new (std::nothrow) float[steps + 1];
  if (!sig) return fail(KLEIN_ERR_INVALID_ARG, "out of host memory");
  rc = klein_sigma_schedule(steps, shift, sig);
  if (rc) {
    delete[] sig;
    return rc;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const StackWs w = carve_stack(ws, seq->batch, nt, ni, nr);
  const bool distilled = m->d.tt_mlp1 != nullptr;
  const long long n = (long long)ni * kLatent;
  const int pi = prof_begin(kProfOther, s);
  if (launch_positions(w.pos, seq->n_txt, seq->img_h, seq->img_w, seq->n_refs, seq->ref_h, seq->ref_w, s) ||
      launch_rope_table(w.pos, w.rope, nt, 10000.f, s)) {
    delete[] sig;
    return cuda_fail("positions / rope table");
  }
  prof_end(pi, s);
  // the text does not change across steps: project it once
  if (m->d.txt_in && (rc = project_text(m, text, seq, w, s))) {
    delete[] sig;
    return rc;
  }
  for (int i = 0; i < steps && rc == KLEIN_OK; ++i) {
    // base model: the text and reference streams' stage 1 is computed once
    const int cache = distilled ? kCacheNone : (i == 0 ? kCacheStore : kCacheLoad);
    rc = stack_impl(m, latents, text, refs, sig[i], distilled ? sig[i + 1] : 0.f, seq, w.v, w, ni, nr, nt, true, cache,
                    s);
    if (rc) break;
    const float dsig = static_cast<float>(static_cast<double>(sig[i + 1]) - static_cast<double>(sig[i]));
    // x0 preview of this step (before its update): every step's, or the last one's
    float* x0 = !x0_out ? nullptr : (x0_every_step ? x0_out + (size_t)i * n : (i == steps - 1 ? x0_out : nullptr));
    const int pi = prof_begin(kProfEuler, s);
    if (launch_euler(latents, w.v, guided ? w.v + n : nullptr, n, dsig, cfg, x0, sig[i], s))
      rc = cuda_fail("euler launch");
    prof_end(pi, s);
  }
  delete[] sig;
  return rc;
}

int klein_op_modln(const void* x, int batch, int n_total, int row0, int rows, int n_txt, int n_img,
                   const float* mod, long long mod_stride, int single_mode, void* h, void* stream) {
  if (!x || !mod || !h) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(x) || !aligned16(mod) || !aligned16(h) || (mod_stride % 4) != 0)
    return fail(KLEIN_ERR_ALIGN, "pointers must be 16-byte aligned, mod_stride a multiple of 4");
  if (batch < 1 || rows < 1 || row0 < 0 || row0 + rows > n_total) return fail(KLEIN_ERR_SHAPE, "bad row range");
  if (launch_modln(static_cast<const float*>(x), n_total, row0, static_cast<__nv_bfloat16*>(h), batch, rows,
                   n_txt, n_img, mod, mod_stride, single_mode, static_cast<cudaStream_t>(stream)))
    return cuda_fail("modln launch");
  return KLEIN_OK;
}

int klein_op_rope_table(const float* pos, int rows, float theta, void* table, void* stream) {
  if (!pos || !table) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (rows < 1 || !(theta > 0.f)) return fail(KLEIN_ERR_SHAPE, "rows must be >= 1, theta > 0");
  if (launch_rope_table(pos, static_cast<float2*>(table), rows, theta, static_cast<cudaStream_t>(stream)))
    return cuda_fail("rope table launch");
  return KLEIN_OK;
}

int klein_op_rope(const void* in, void* out, const void* table, int rows, int heads, void* stream) {
  if (!in || !out || !table) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(in) || !aligned16(out) || !aligned16(table)) return fail(KLEIN_ERR_ALIGN, "unaligned pointer");
  if (rows < 1 || heads < 1) return fail(KLEIN_ERR_SHAPE, "rows and heads must be >= 1");
  if (launch_rope_apply(static_cast<const __nv_bfloat16*>(in), static_cast<__nv_bfloat16*>(out),
                        static_cast<const float2*>(table), rows, heads, static_cast<cudaStream_t>(stream)))
    return cuda_fail("rope launch");
  return KLEIN_OK;
}

int klein_op_euler(float* x, const float* v_cond, const float* v_uncond, long long n, float dsigma, float g,
                   float* x0_out, float sigma, void* stream) {
  if (!x || !v_cond) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(x) || !aligned16(v_cond) || (v_uncond && !aligned16(v_uncond)) || (x0_out && !aligned16(x0_out)))
    return fail(KLEIN_ERR_ALIGN, "unaligned pointer");
  if (n < 0 || (n % 4) != 0) return fail(KLEIN_ERR_SHAPE, "n must be a non-negative multiple of 4");
  if (launch_euler(x, v_cond, v_uncond, n, dsigma, g, x0_out, sigma, static_cast<cudaStream_t>(stream)))
    return cuda_fail("euler launch");
  return KLEIN_OK;
}

int klein_op_gemm(const void* a, const void* b, float* c, int m, int n, int k, void* stream) {
  if (!a || !b || !c) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(a) || !aligned16(b) || !aligned16(c)) return fail(KLEIN_ERR_ALIGN, "unaligned pointer");
  if (m < 1 || n < 128 || (n % 128) != 0 || k < 64 || (k % 64) != 0)
    return fail(KLEIN_ERR_SHAPE, "need M >= 1, N a multiple of 128, K a multiple of 64");
  CUtensorMap ma, mb;
  if (make_map_3d(&ma, a, k, m, 1, (uint64_t)k * 2, (uint64_t)m * k * 2, 64, 128) ||
      make_map_2d(&mb, b, k, n, (uint64_t)k * 2, 64, 128))
    return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  // N a multiple of 256: the block GEMM configuration (CTA pairs unless
  // built without them); otherwise single CTAs with 128-column tiles.
  const bool wide = (n % 256) == 0;
  const int rows_per_tile = wide ? kGemmRowsPerTile : 128;
  GemmArgs g{};
  g.batch = 1;
  g.rows = m;
  g.m_tiles_per_b = (m + rows_per_tile - 1) / rows_per_tile;
  g.n_tiles = n / (wide ? 256 : 128);
  g.k_blocks = k / 64;
  g.out = c;
  g.out_ld = n;
  g.out_bstride = m;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rc = wide ? launch_block_gemm(kEpiF32, ma, mb, g, s) : launch_gemm(128, kEpiF32, ma, mb, g, s);
  if (rc) return cuda_fail("gemm launch");
  return KLEIN_OK;
}

int klein_op_gemm_e4m3(const void* a, const float* a_scale, const void* b, const float* b_scale, float* c, int m,
                       int n, int k, void* stream) {
  if (!a || !a_scale || !b || !b_scale || !c) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(a) || !aligned16(b) || !aligned16(c) || !aligned16(a_scale) || !aligned16(b_scale))
    return fail(KLEIN_ERR_ALIGN, "unaligned pointer");
  if (m < 1 || n < 256 || (n % 256) != 0 || k < 128 || (k % 128) != 0)
    return fail(KLEIN_ERR_SHAPE, "need M >= 1, N a multiple of 256, K a multiple of 128");
  CUtensorMap ma, mb;
  if (make_map_3d(&ma, a, k, m, 1, (uint64_t)k, (uint64_t)m * k, 128, 128, 1) ||
      make_map_2d(&mb, b, k, n, (uint64_t)k, 128, 128, 1))
    return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  GemmArgs g{};
  g.batch = 1;
  g.rows = m;
  g.m_tiles_per_b = (m + 255) / 256;
  g.n_tiles = n / 256;
  g.k_blocks = k / 128;
  g.out = c;
  g.out_ld = n;
  g.out_bstride = m;
  g.a_scale = a_scale;
  g.b_scale = b_scale;
  if (launch_gemm_pair(kEpiF32, ma, mb, g, static_cast<cudaStream_t>(stream), 1)) return cuda_fail("gemm launch");
  return KLEIN_OK;
}

int klein_quantize_rowwise_e4m3(const void* src, long long rows, int cols, void* codes, float* scale,
                                void* stream) {
  if (!src || !codes || !scale) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(src) || !aligned16(codes) || !aligned16(scale)) return fail(KLEIN_ERR_ALIGN, "unaligned pointer");
  if (rows < 1 || rows > 0x7fffffffLL || cols < 8 || (cols % 8) != 0 || cols > kOutK)
    return fail(KLEIN_ERR_SHAPE, "need rows >= 1 and cols a multiple of 8 in [8, 12288]");
  const char* s0 = static_cast<const char*>(src);
  const char* c0 = static_cast<const char*>(codes);
  if (c0 < s0 + rows * cols * 2 && s0 < c0 + rows * cols)
    return fail(KLEIN_ERR_INVALID_ARG, "codes overlap src");
  if (launch_quantize_rows(static_cast<const __nv_bfloat16*>(src), cols, static_cast<uint8_t*>(codes), cols, scale,
                           rows, cols, static_cast<cudaStream_t>(stream)))
    return cuda_fail("quantisation launch");
  return KLEIN_OK;
}

int klein_op_modln_e4m3(const void* x, int batch, int n_total, int row0, int rows, int n_txt, int n_img,
                        const float* mod, long long mod_stride, void* codes, float* scale, void* stream) {
  if (!x || !mod || !codes || !scale) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(x) || !aligned16(mod) || !aligned16(codes) || !aligned16(scale) || (mod_stride % 4) != 0)
    return fail(KLEIN_ERR_ALIGN, "pointers must be 16-byte aligned, mod_stride a multiple of 4");
  if (batch < 1 || rows < 1 || row0 < 0 || row0 + rows > n_total) return fail(KLEIN_ERR_SHAPE, "bad row range");
  if (launch_modln_e4m3(static_cast<const float*>(x), n_total, row0, static_cast<uint8_t*>(codes), scale, batch,
                        rows, n_txt, n_img, mod, mod_stride, static_cast<cudaStream_t>(stream)))
    return cuda_fail("modln launch");
  return KLEIN_OK;
}

int klein_quantize_nvfp4(const void* src, long long rows, int cols, int mode, void* codes, void* sf, float* g,
                         void* stream) {
  if (!src || !codes || !sf || !g) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(src) || !aligned16(codes) || !aligned16(sf) || !aligned16(g))
    return fail(KLEIN_ERR_ALIGN, "unaligned pointer");
  if (mode < KLEIN_NVFP4_MATRIX || mode > KLEIN_NVFP4_IN_PROJ) return fail(KLEIN_ERR_INVALID_ARG, "bad mode");
  if (rows < 1 || rows > (1 << 30) || cols < 64 || (cols % 64) != 0 || cols > kOutK)
    return fail(KLEIN_ERR_SHAPE, "need rows >= 1 and cols a multiple of 64 in [64, 12288]");
  if (mode == KLEIN_NVFP4_IN_PROJ && (rows != kInCols || cols != kDim))
    return fail(KLEIN_ERR_SHAPE, "the in-projection order needs a [27648][3072] matrix");
  const char* s0 = static_cast<const char*>(src);
  const char* c0 = static_cast<const char*>(codes);
  if (c0 < s0 + rows * cols * 2 && s0 < c0 + rows * cols / 2) return fail(KLEIN_ERR_INVALID_ARG, "codes overlap src");
  const bool per_row = mode == KLEIN_NVFP4_ROWS;
  const int rows_pad = round_up(static_cast<int>(rows), per_row ? 256 : 128);
  if (launch_quantize_nvfp4(static_cast<const __nv_bfloat16*>(src), cols, mode == KLEIN_NVFP4_IN_PROJ,
                            static_cast<uint8_t*>(codes), cols / 2, static_cast<uint8_t*>(sf), per_row ? g : nullptr,
                            per_row ? nullptr : g, 1, static_cast<int>(rows), rows_pad, cols,
                            static_cast<cudaStream_t>(stream)))
    return cuda_fail("quantisation launch");
  return KLEIN_OK;
}

int klein_op_modln_nvfp4(const void* x, int batch, int n_total, int row0, int rows, int n_txt, int n_img,
                         const float* mod, long long mod_stride, void* codes, void* sf, float* g, void* stream) {
  if (!x || !mod || !codes || !sf || !g) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(x) || !aligned16(mod) || !aligned16(codes) || !aligned16(sf) || !aligned16(g) || (mod_stride % 4) != 0)
    return fail(KLEIN_ERR_ALIGN, "pointers must be 16-byte aligned, mod_stride a multiple of 4");
  if (batch < 1 || rows < 1 || row0 < 0 || row0 + rows > n_total) return fail(KLEIN_ERR_SHAPE, "bad row range");
  if (launch_modln_nvfp4(static_cast<const float*>(x), n_total, row0, static_cast<uint8_t*>(codes),
                         static_cast<uint8_t*>(sf), g, batch, rows, n_txt, n_img, mod, mod_stride,
                         static_cast<cudaStream_t>(stream)))
    return cuda_fail("modln launch");
  return KLEIN_OK;
}

int klein_op_gemm_nvfp4(const void* a, const void* a_sf, const float* a_g, const void* b, const void* b_sf,
                        const float* b_g, float* c, int m, int n, int k, void* stream) {
  if (!a || !a_sf || !a_g || !b || !b_sf || !b_g || !c) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(a) || !aligned16(a_sf) || !aligned16(a_g) || !aligned16(b) || !aligned16(b_sf) || !aligned16(b_g) ||
      !aligned16(c))
    return fail(KLEIN_ERR_ALIGN, "unaligned pointer");
  if (m < 1 || n < 128 || (n % 128) != 0 || k < 256 || (k % 256) != 0)
    return fail(KLEIN_ERR_SHAPE, "need M >= 1, N a multiple of 128, K a multiple of 256");
  GemmArgs g{};
  g.batch = 1;
  g.rows = m;
  g.m_tiles_per_b = (m + 255) / 256;
  g.n_tiles = n / 128;
  g.k_blocks = k / 256;
  g.out = c;
  g.out_ld = n;
  g.out_bstride = m;
  g.a_scale = a_g;
  g.b_g = b_g;
  const int rc = launch_gemm_nvfp4(kEpiF32, a, k / 2, a_sf, b, b_sf, g, n, static_cast<cudaStream_t>(stream));
  if (rc == -2) return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  if (rc) return cuda_fail("gemm launch");
  return KLEIN_OK;
}

int klein_op_attention(const void* q, const void* k, const void* vt, int batch, int rows, int rows_pad, void* out,
                       long long out_ld, void* stream) {
  if (!q || !k || !vt || !out) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(vt) || !aligned16(out) || (out_ld % 8) != 0)
    return fail(KLEIN_ERR_ALIGN, "unaligned pointer or out_ld");
  if (batch < 1 || rows < 1 || rows_pad < rows || (rows_pad % 8) != 0 || out_ld < kDim)
    return fail(KLEIN_ERR_SHAPE, "bad attention shape");
  AttnArgs at{};
  at.batch = batch;
  at.heads = kHeads;
  at.rows = rows;
  at.rows_pad = rows_pad;
  at.q = static_cast<const __nv_bfloat16*>(q);
  at.k = static_cast<const __nv_bfloat16*>(k);
  at.vt = static_cast<const __nv_bfloat16*>(vt);
  at.out = static_cast<__nv_bfloat16*>(out);
  at.out_ld = out_ld;
  at.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(128.0));
  const int arc = launch_attention(at, static_cast<cudaStream_t>(stream));
  if (arc == -2) return fail(KLEIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  if (arc) return cuda_fail("attention launch");
  return KLEIN_OK;
}

}  // extern "C"
