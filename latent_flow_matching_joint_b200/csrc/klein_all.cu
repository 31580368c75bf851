// Single translation unit of the Klein library: the kernels share the
// device error word and wait limit defined in klein_capi.cu, so they are
// compiled together (no relocatable device code needed).
#include "kernels_mem.cu"
#include "gemm.cu"
#include "attention.cu"
#include "nvfp4.cu"
#include "klein_capi.cu"
#include "static_ws.cu"
