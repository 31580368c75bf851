// klein_block_forward_static: the block forward for callers that cannot
// allocate device memory. Its scratch (the bf16 modulated input, q, k, v^T,
// the attention|SwiGLU operand of the out-projection and the RoPE table)
// lives in one fixed array in this library's own device memory instead of a
// caller-supplied workspace. The array is a file-scope __device__ object, so
// every GPU that loads the library holds it until the process exits.
#include "../../include/klein.h"
#include "common.cuh"
#include "internal.h"

namespace klein {

// Largest batch * round_up(rows, 128) the fixed scratch can hold.
constexpr int kStaticMaxRows = 256;
// Bytes of carve_block(batch, rows) for every batch * round_up(rows, 128) <=
// kStaticMaxRows: h, q, k, v^T, attention|SwiGLU operand, RoPE table, the two
// per-row scale vectors, and the NVFP4 block scales of the two GEMM inputs,
// laid out per batch item over round_up(rows, 256) rows (at most 2 *
// kStaticMaxRows rows in all). Every region is a multiple of 256 bytes.
constexpr size_t kStaticWsBytes = (size_t)kStaticMaxRows * kDim * 2 +
                                  3 * (size_t)kHeads * kStaticMaxRows * kHeadDim * 2 +
                                  (size_t)kStaticMaxRows * kOutK * 2 + (size_t)kStaticMaxRows * kPairs * sizeof(float2) +
                                  2 * (size_t)kStaticMaxRows * sizeof(float) +
                                  2 * (size_t)kStaticMaxRows * (kDim / 16 + kOutK / 16);

static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

// Device address of g_static_ws per device, looked up on the first call made
// with that device current. In host code the symbol is only a host-side
// stand-in; the kernels must be given this device address.
static void* g_static_ws_addr[64] = {};

static int static_ws_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(KLEIN_ERR_UNSUPPORTED, "device index %d out of range", dev);
  if (!g_static_ws_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_ws);
    if (e != cudaSuccess || p == nullptr)
      return fail(KLEIN_ERR_CUDA, "cudaGetSymbolAddress of the fixed scratch: %s", cudaGetErrorString(e));
    g_static_ws_addr[dev] = p;
  }
  *out = g_static_ws_addr[dev];
  return KLEIN_OK;
}

}  // namespace klein

extern "C" int klein_block_forward_static(const klein_block_weights* w, void* x, int batch, int n_total, int row0,
                                          int rows, int n_txt, int n_img, const float* pos, const float* mod,
                                          void* stream) {
  using namespace klein;
  int rc = check_block_weights(w);
  if (rc) return rc;
  if (!x || !pos || !mod) return fail(KLEIN_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(x) || !aligned16(pos) || !aligned16(mod))
    return fail(KLEIN_ERR_ALIGN, "pointers must be 16-byte aligned");
  if ((rc = check_block_rows(batch, n_total, row0, rows, n_txt, n_img))) return rc;
  const long long need_rows = (long long)batch * round_up(rows, 128);
  if (need_rows > kStaticMaxRows)
    return fail(KLEIN_ERR_WORKSPACE,
                "batch * rows rounded up to 128 is %lld; the fixed scratch of klein_block_forward_static holds %d "
                "(use klein_block_forward with a workspace)",
                need_rows, kStaticMaxRows);
  void* scratch = nullptr;
  rc = static_ws_address(&scratch);
  if (rc) return rc;
  const BlockWs bw = carve_block(scratch, batch, rows);
  if (bw.bytes > kStaticWsBytes) return fail(KLEIN_ERR_WORKSPACE, "fixed scratch too small (%zu bytes)", bw.bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_rope_table(pos + (size_t)row0 * 4, bw.rope, rows, 10000.f, s)) return cuda_fail("rope table");
  return block_impl(w, static_cast<float*>(x), batch, n_total, row0, rows, n_txt, n_img, bw.rope, mod, bw, s);
}
