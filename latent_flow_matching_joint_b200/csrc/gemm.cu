// Persistent tcgen05 GEMM, C = A * B^T, bf16 operands, fp32 accumulation in
// tensor memory, fed by TMA, with the block's fused epilogues. The CTA-pair
// variant also runs rowwise-scaled e4m3 operands (kind::f8f6f4) for the FP8
// block: same shared-memory bytes per stage (128 K elements instead of 64),
// twice the MMA rate, and the two scales applied in the epilogue.
//
// Roles of the single-CTA kernel (192 threads, one CTA per SM):
//   warp 0      TMA producer: A tile 128 x 64 and B tile BN x 64 per stage
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2..5  epilogue: one accumulator row per thread (TMEM lane quarter
//               = warp % 4), two accumulator buffers so that the epilogue of
//               tile i overlaps the main loop of tile i+1.
// The CTA-pair kernel below has the same roles with eight epilogue warps
// (320 threads): two per lane quarter, each with half of the tile's columns.
// Tiles are visited M-fastest (the CTAs in flight share B tiles in L2 while A
// stays resident) or N-fastest (B stays resident in L2, each A row block is
// read from HBM once), whichever operand fits in L2.
//
// Epilogues (FLUX.3 Klein block, Diffusers release blog "Speed,
// architecture, and how the tokens move", and its Chinese translation's
// block pseudo-code):
//   kEpiQKV   in-projection: q and k are RMS-normalised per head and rotated
//             by the 4-axis RoPE, v is stored transposed for the attention
//             kernel, and the paired gate|up tiles leave silu(gate) * up.
//   kEpiResid out-projection: x += gate[mode(row)] * (attn + mlp).
#include "common.cuh"
#include "internal.h"

// Epilogue warps of the CTA-pair kernel: 8 (two per TMEM lane quarter), or 4
// (one per quarter; measured 3 % slower on the FP8 block, the same on bf16).
#ifndef KLEIN_PAIR_EPI_WARPS
#define KLEIN_PAIR_EPI_WARPS 8
#endif

namespace klein {

template <int BN>
struct GemmCfg {
  static constexpr int kStageA = 128 * 64 * 2;
  static constexpr int kStageB = BN * 64 * 2;
  static constexpr int kStage = kStageA + kStageB;
  static constexpr int kStages = (BN == 256) ? 4 : 6;
  static constexpr int kTileBytes = kStages * kStage;
  static constexpr int kSmem = kTileBytes + 1024 + 256;
  static constexpr uint32_t kTmemCols = 2 * BN;
  static constexpr int kThreads = 192;
};

static constexpr float kRmsEps = 1e-6f;

__device__ __forceinline__ void store16(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  *reinterpret_cast<uint4*>(p) = make_uint4(a, b, c, d);
}

// ---- epilogues: one thread = one accumulator row; taddr = lane quarter base

// e4m3 operands: the accumulator holds sum(code_a * code_b); the value is that
// times the row's activation scale and the output channel's weight scale.
__device__ __forceinline__ void dequant32(float* v, float sa, const float* sb) {
  const float4* s4 = reinterpret_cast<const float4*>(sb);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 t = __ldg(s4 + i);
    v[4 * i + 0] *= sa * t.x;
    v[4 * i + 1] *= sa * t.y;
    v[4 * i + 2] *= sa * t.z;
    v[4 * i + 3] *= sa * t.w;
  }
}

// part / nparts: this warp's share of the tile's columns when several
// epilogue warps serve the same TMEM lane quarter.
// The output channel's weight scale alone (the row's scale folded elsewhere).
__device__ __forceinline__ void colscale32(float* v, const float* sb) {
  const float4* s4 = reinterpret_cast<const float4*>(sb);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 t = __ldg(s4 + i);
    v[4 * i + 0] *= t.x;
    v[4 * i + 1] *= t.y;
    v[4 * i + 2] *= t.z;
    v[4 * i + 3] *= t.w;
  }
}

template <int BN, bool F8>
__device__ __forceinline__ void epi_store(uint32_t taddr, const GemmArgs& g, int b, int r, int n_idx, bool f32,
                                          int part, int nparts) {
  const bool valid = r < g.rows;
  const float sa = F8 && valid ? __ldg(g.a_scale + (long long)b * g.rows + r) : 0.f;
  float v[32];
  const int per = BN / 32 / nparts;
#pragma unroll 1
  for (int c = part * per; c < (part + 1) * per; ++c) {
    tmem_ld32(taddr + 32 * c, v);
    if (!valid) continue;
    if (F8) dequant32(v, sa, g.b_scale + n_idx * BN + 32 * c);
    const int col = n_idx * BN + 32 * c;
    const int copies = g.replicate > 1 ? g.replicate : 1;
    for (int rep = 0; rep < copies; ++rep) {
      const int bb = g.replicate > 1 ? rep : b;
      const long long orow = (long long)bb * g.out_bstride + g.out_row0 + r;
      if (f32) {
        float* o = reinterpret_cast<float*>(g.out) + orow * g.out_ld + col;
#pragma unroll
        for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(o + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      } else {
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(g.out) + orow * g.out_ld + col;
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          store16(o + i, pack_bf16(v[i], v[i + 1]), pack_bf16(v[i + 2], v[i + 3]), pack_bf16(v[i + 4], v[i + 5]),
                  pack_bf16(v[i + 6], v[i + 7]));
      }
    }
  }
}

template <bool F8>
__device__ __forceinline__ void epi_qkv(uint32_t taddr, const GemmArgs& g, int b, int r, int n_idx, int part,
                                        int nparts) {
  const bool valid = r < g.rows;
  const float sa = F8 && valid ? __ldg(g.a_scale + (long long)b * g.rows + r) : 0.f;
  float v[32];
  if (n_idx < g.b_split) {
    const int which = n_idx / 12;            // 0 q, 1 k, 2 v
    const int head0 = (n_idx % 12) * 2;
#pragma unroll 1
    for (int hh = part; hh < 2; hh += nparts) {
      const int head = head0 + hh;
      const uint32_t tcol = taddr + hh * 128;
      const long long bh = (long long)b * kHeads + head;
      const float* sb = F8 ? g.b_scale + n_idx * 256 + hh * 128 : nullptr;
      if (which == 2) {
        __nv_bfloat16* dst = g.vt + bh * kHeadDim * g.rows_pad + r;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(tcol + 32 * c, v);
          if (F8) dequant32(v, sa, sb + 32 * c);
          if (valid) {
#pragma unroll
            for (int i = 0; i < 32; ++i) dst[(long long)(32 * c + i) * g.rows_pad] = __float2bfloat16_rn(v[i]);
          }
        }
        continue;
      }
      const float* w = which == 0 ? g.q_norm : g.k_norm;
      __nv_bfloat16* dst = (which == 0 ? g.q : g.k) + (bh * g.rows_pad + r) * kHeadDim;
      // e4m3: the head's values are sa * acc * sb; the row scale sa is folded
      // into the RMS normalisation (sa * rsqrt(sa^2 * mean((acc sb)^2) + eps))
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tcol + 32 * c, v);
        if (F8) colscale32(v, sb + 32 * c);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
      }
      const float rs = F8 ? sa * rsqrtf(sa * sa * ss * (1.0f / kHeadDim) + kRmsEps)
                          : rsqrtf(ss * (1.0f / kHeadDim) + kRmsEps);
      // (cos, sin) of two pairs and four norm weights per 16-byte load
      const float4* rope4 = reinterpret_cast<const float4*>(g.rope + (long long)(valid ? r : 0) * kPairs);
      const float4* w4 = reinterpret_cast<const float4*>(w);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tcol + 32 * c, v);
        if (!valid) continue;
        if (F8) colscale32(v, sb + 32 * c);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const int d = 32 * c + i;
          const float4 wn = __ldg(w4 + (d >> 2));
          const float4 cs = __ldg(rope4 + (d >> 2));  // pairs d/2 and d/2 + 1
          const float y0 = v[i] * rs * wn.x, y1 = v[i + 1] * rs * wn.y;
          const float y2 = v[i + 2] * rs * wn.z, y3 = v[i + 3] * rs * wn.w;
          pk[i >> 1] = pack_bf16(y0 * cs.x - y1 * cs.y, y0 * cs.y + y1 * cs.x);
          pk[(i >> 1) + 1] = pack_bf16(y2 * cs.z - y3 * cs.w, y2 * cs.w + y3 * cs.z);
        }
        __nv_bfloat16* o = dst + 32 * c;
        store16(o, pk[0], pk[1], pk[2], pk[3]);
        store16(o + 8, pk[4], pk[5], pk[6], pk[7]);
        store16(o + 16, pk[8], pk[9], pk[10], pk[11]);
        store16(o + 24, pk[12], pk[13], pk[14], pk[15]);
      }
    }
  } else {
    const int chunk = n_idx - g.b_split;     // 128 hidden units: gate cols 0..127, up cols 128..255
    __nv_bfloat16* dst = g.a_out + ((long long)b * g.rows + r) * kOutK + kDim + chunk * 128;
    float u[32];
    const int per = 4 / nparts;
#pragma unroll 1
    for (int c = part * per; c < (part + 1) * per; ++c) {
      tmem_ld32(taddr + 32 * c, v);
      tmem_ld32(taddr + 128 + 32 * c, u);
      if (!valid) continue;
      if (F8) {
        dequant32(v, sa, g.b_scale + 3 * kDim + chunk * 128 + 32 * c);
        dequant32(u, sa, g.b_scale + 3 * kDim + kMlp + chunk * 128 + 32 * c);
      }
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) pk[i >> 1] = pack_bf16(silu(v[i]) * u[i], silu(v[i + 1]) * u[i + 1]);
      __nv_bfloat16* o = dst + 32 * c;
      store16(o, pk[0], pk[1], pk[2], pk[3]);
      store16(o + 8, pk[4], pk[5], pk[6], pk[7]);
      store16(o + 16, pk[8], pk[9], pk[10], pk[11]);
      store16(o + 24, pk[12], pk[13], pk[14], pk[15]);
    }
  }
}

template <int BN, bool F8>
__device__ __forceinline__ void epi_resid(uint32_t taddr, const GemmArgs& g, int b, int r, int n_idx, int part,
                                          int nparts) {
  const bool valid = r < g.rows;
  const float sa = F8 && valid ? __ldg(g.a_scale + (long long)b * g.rows + r) : 0.f;
  const int grow = g.x_row0 + r;
  const int mode = mode_of_row(grow, g.n_txt, g.n_img);
  const float* gate = g.mod + (long long)mode * 3 * kDim + 2 * kDim + n_idx * BN;
  float* xr = g.x + ((long long)b * g.x_bstride + grow) * kDim + n_idx * BN;
  float v[32];
  const int per = BN / 32 / nparts;
#pragma unroll 1
  for (int c = part * per; c < (part + 1) * per; ++c) {
    tmem_ld32(taddr + 32 * c, v);
    if (!valid) continue;
    if (F8) dequant32(v, sa, g.b_scale + n_idx * BN + 32 * c);
    float4* p = reinterpret_cast<float4*>(xr + 32 * c);
    const float4* gt = reinterpret_cast<const float4*>(gate + 32 * c);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 xv = p[i];
      const float4 gv = __ldg(gt + i);
      xv.x = fmaf(gv.x, v[4 * i + 0], xv.x);
      xv.y = fmaf(gv.y, v[4 * i + 1], xv.y);
      xv.z = fmaf(gv.z, v[4 * i + 2], xv.z);
      xv.w = fmaf(gv.w, v[4 * i + 3], xv.w);
      p[i] = xv;
    }
  }
}

// ---- the kernel

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const GemmArgs g) {
  using Cfg = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kTileBytes);
  uint64_t* empty = full + Cfg::kStages;
  uint64_t* acc_full = empty + Cfg::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // operands and outputs are touched only after the previous kernel completes

  const int m_tiles = g.batch * g.m_tiles_per_b;
  const int total = m_tiles * g.n_tiles;
  constexpr uint32_t idesc = idesc_bf16_f32(128, BN);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      StageLog log;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const int m_idx = g.n_fastest ? tile / g.n_tiles : tile % m_tiles;
        const int n_idx = g.n_fastest ? tile % g.n_tiles : tile / m_tiles;
        const int b = m_idx / g.m_tiles_per_b;
        const int row0 = (m_idx % g.m_tiles_per_b) * 128;
        int brow0, brow1;
        if (EPI == kEpiQKV && n_idx >= g.b_split) {
          const int chunk = n_idx - g.b_split;
          brow0 = 3 * kDim + chunk * 128;
          brow1 = 3 * kDim + kMlp + chunk * 128;
        } else {
          brow0 = n_idx * BN;
          brow1 = brow0 + 128;
        }
        bool ok = true;
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, 0x101)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], Cfg::kStage);
          log.armed(stage, phase);
          uint8_t* sa = smem + stage * Cfg::kStage;
          uint8_t* sb = sa + Cfg::kStageA;
          tma_load_3d(sa, &map_a, &full[stage], kb * 64, row0, b);
          tma_load_2d(sb, &map_b, &full[stage], kb * 64, brow0);
          if (BN == 256) tma_load_2d(sb + 128 * 128, &map_b, &full[stage], kb * 64, brow1);
          if (++stage == Cfg::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
      log.drain(full, Cfg::kStages, 0x105);  // no TMA write may land after the CTA exits
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, 0x102)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, 0x103)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * Cfg::kStage);
          const uint32_t b0 = a0 + Cfg::kStageA;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(d, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc, (kb | k) != 0);
          umma_commit(&empty[stage]);
          if (++stage == Cfg::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
      }
      // every MMA issued here has completed before TMEM is freed
      umma_commit(drain);
      mbar_wait(drain, 0, 0x106);
    }
  } else {
    const int quarter = warp & 3;
    const int rloc = quarter * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      const int m_idx = g.n_fastest ? tile / g.n_tiles : tile % m_tiles;
      const int n_idx = g.n_fastest ? tile % g.n_tiles : tile / m_tiles;
      const int b = m_idx / g.m_tiles_per_b;
      const int r = (m_idx % g.m_tiles_per_b) * 128 + rloc;
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(&acc_full[acc], acc_phase, 0x104)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + acc * BN + (static_cast<uint32_t>(quarter * 32) << 16);
      if (EPI == kEpiF32) epi_store<BN, false>(taddr, g, b, r, n_idx, true, 0, 1);
      else if (EPI == kEpiBF16) epi_store<BN, false>(taddr, g, b, r, n_idx, false, 0, 1);
      else if (EPI == kEpiQKV) epi_qkv<false>(taddr, g, b, r, n_idx, 0, 1);
      else epi_resid<BN, false>(taddr, g, b, r, n_idx, 0, 1);
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

template <int BN, int EPI>
static int launch_one(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g, cudaStream_t s) {
  using Cfg = GemmCfg<BN>;
  static bool configured[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return -1;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(gemm_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem) !=
        cudaSuccess)
      return -1;
    configured[dev] = true;
  }
  const int total = g.batch * g.m_tiles_per_b * g.n_tiles;
  if (total <= 0) return 0;
  const int grid = total < num_sms() ? total : num_sms();
  const cudaError_t e = launch_kernel(gemm_kernel<BN, EPI>, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmem, s, 1, ma, mb, g);
  note_launch();
  return (e == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

// ---- CTA-pair variant: 256 x 256 output tiles per cluster of 2 CTAs.
// Each CTA loads its 128 rows of A and its 128 rows of B (half the N tile) per
// stage, so operand bytes per FLOP from L2 drop by a third against the
// single-CTA 128 x 256 tile. The even CTA issues cta_group::2 MMAs
// (M = 256, N = 256) that read both CTAs' shared memory and write each CTA's
// 128 accumulator rows into its own tensor memory; its commits arrive on the
// barriers of both CTAs. TMA completions of both CTAs are counted on the even
// CTA's full barrier; both CTAs' epilogue threads release the accumulator on
// the even CTA's empty barrier.

struct PairCfg {
  static constexpr int kStageA = 128 * 64 * 2;
  static constexpr int kStageB = 128 * 64 * 2;
  static constexpr int kStage = kStageA + kStageB;
  static constexpr int kStages = 6;  // 7 (the most that fits) measured 1 % slower
  static constexpr int kTileBytes = kStages * kStage;
  static constexpr int kSmem = kTileBytes + 1024 + 256;
  static constexpr uint32_t kTmemCols = 512;  // two 256-column accumulators
  // Epilogue warps: two per TMEM lane quarter, each taking half of the
  // tile's columns, so that one warp's TMEM and global latencies overlap the
  // other's work (the e4m3 main loop is short enough to wait on a single
  // warp per quarter).
  static constexpr int kEpiWarps = KLEIN_PAIR_EPI_WARPS;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
};

template <int EPI, bool F8>
__global__ void __launch_bounds__(PairCfg::kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                     const GemmArgs g) {
  using Cfg = PairCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kTileBytes);
  uint64_t* empty = full + Cfg::kStages;
  uint64_t* acc_full = empty + Cfg::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * 32 * Cfg::kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barrier initialisation and the TMEM allocation are visible pair-wide
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // operands and outputs are touched only after the previous kernel completes

  const int m_tiles = g.batch * g.m_tiles_per_b;
  const int total = m_tiles * g.n_tiles;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(256, 256) : idesc_bf16_f32(256, 256);
  constexpr int kBlockK = F8 ? 128 : 64;  // elements per 128-byte swizzle row

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      StageLog log;
      for (int tile = pair; tile < total; tile += npairs) {
        const int m_idx = g.n_fastest ? tile / g.n_tiles : tile % m_tiles;
        const int n_idx = g.n_fastest ? tile % g.n_tiles : tile / m_tiles;
        const int b = m_idx / g.m_tiles_per_b;
        const int row0 = (m_idx % g.m_tiles_per_b) * 256 + 128 * static_cast<int>(rank);
        int brow;
        if (EPI == kEpiQKV && n_idx >= g.b_split) {
          const int chunk = n_idx - g.b_split;
          brow = (leader ? 3 * kDim : 3 * kDim + kMlp) + chunk * 128;
        } else {
          brow = n_idx * 256 + 128 * static_cast<int>(rank);
        }
        bool ok = true;
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, 0x111)) { ok = false; break; }
          if (leader) {
            mbar_arrive_expect_tx(&full[stage], 2 * Cfg::kStage);
            log.armed(stage, phase);
          }
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
          uint8_t* sa = smem + stage * Cfg::kStage;
          tma_load_3d_pair(sa, &map_a, bar, kb * kBlockK, row0, b);
          tma_load_2d_pair(sa + Cfg::kStageA, &map_b, bar, kb * kBlockK, brow);
          if (++stage == Cfg::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
      // The even CTA's full barriers count the bytes of both CTAs' loads:
      // once every phase it armed is complete, no TMA write of the pair is
      // still in flight (the cluster barrier below keeps the odd CTA alive
      // until then).
      if (leader) log.drain(full, Cfg::kStages, 0x115);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int tile = pair; tile < total; tile += npairs, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, 0x112)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * 256;
        bool ok = true;
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, 0x113)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * Cfg::kStage);
          const uint32_t b0 = a0 + Cfg::kStageA;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (F8) umma_e4m3_pair(d, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc, (kb | k) != 0);
            else umma_bf16_pair(d, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc, (kb | k) != 0);
          }
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == Cfg::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair(&acc_full[acc], 0x3);
      }
      // every pair MMA issued here has completed before either CTA frees its TMEM
      umma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, 0x116);
    }
  } else {
    const int quarter = warp & 3;
    const int rloc = quarter * 32 + lane;
    const int nparts = Cfg::kEpiWarps / 4;
    const int part = (warp - 2) / 4;
    int it = 0;
    for (int tile = pair; tile < total; tile += npairs, ++it) {
      const int m_idx = g.n_fastest ? tile / g.n_tiles : tile % m_tiles;
      const int n_idx = g.n_fastest ? tile % g.n_tiles : tile / m_tiles;
      const int b = m_idx / g.m_tiles_per_b;
      const int r = (m_idx % g.m_tiles_per_b) * 256 + 128 * static_cast<int>(rank) + rloc;
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(&acc_full[acc], acc_phase, 0x114)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + acc * 256 + (static_cast<uint32_t>(quarter * 32) << 16);
      if (EPI == kEpiF32) epi_store<256, F8>(taddr, g, b, r, n_idx, true, part, nparts);
      else if (EPI == kEpiQKV) epi_qkv<F8>(taddr, g, b, r, n_idx, part, nparts);
      else epi_resid<256, F8>(taddr, g, b, r, n_idx, part, nparts);
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[acc]), 0));
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();  // every pair MMA and every epilogue of both CTAs is done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
  }
}

template <int EPI, bool F8>
static int launch_pair_one(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g, cudaStream_t s) {
  using Cfg = PairCfg;
  static int max_pairs_dev[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return -1;
  int& max_pairs = max_pairs_dev[dev];
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(Cfg::kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (max_pairs == 0) {
    if (cudaFuncSetAttribute(gemm_pair_kernel<EPI, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem) !=
        cudaSuccess)
      return -1;
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<EPI, F8>, &cfg) != cudaSuccess || n < 1) return -1;
    max_pairs = n;
  }
  const int total = g.batch * g.m_tiles_per_b * g.n_tiles;
  if (total <= 0) return 0;
  const int pairs = total < max_pairs ? total : max_pairs;
  const cudaError_t e =
      launch_kernel(gemm_pair_kernel<EPI, F8>, dim3(2 * pairs), dim3(Cfg::kThreads), Cfg::kSmem, s, 2, ma, mb, g);
  note_launch();
  return (e == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}

int launch_gemm_pair(int epi, const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g, cudaStream_t s,
                     int e4m3) {
  if (e4m3) {
    if (!g.a_scale || !g.b_scale) return -2;
    switch (epi) {
      case kEpiF32: return launch_pair_one<kEpiF32, true>(ma, mb, g, s);
      case kEpiQKV: return launch_pair_one<kEpiQKV, true>(ma, mb, g, s);
      case kEpiResid: return launch_pair_one<kEpiResid, true>(ma, mb, g, s);
    }
    return -2;
  }
  switch (epi) {
    case kEpiF32: return launch_pair_one<kEpiF32, false>(ma, mb, g, s);
    case kEpiQKV: return launch_pair_one<kEpiQKV, false>(ma, mb, g, s);
    case kEpiResid: return launch_pair_one<kEpiResid, false>(ma, mb, g, s);
  }
  return -2;
}

int launch_gemm(int bn, int epi, const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g,
                cudaStream_t s) {
  if (bn == 256) {
    switch (epi) {
      case kEpiF32: return launch_one<256, kEpiF32>(ma, mb, g, s);
      case kEpiBF16: return launch_one<256, kEpiBF16>(ma, mb, g, s);
      case kEpiQKV: return launch_one<256, kEpiQKV>(ma, mb, g, s);
      case kEpiResid: return launch_one<256, kEpiResid>(ma, mb, g, s);
    }
  } else if (bn == 128) {
    switch (epi) {
      case kEpiF32: return launch_one<128, kEpiF32>(ma, mb, g, s);
      case kEpiBF16: return launch_one<128, kEpiBF16>(ma, mb, g, s);
    }
  }
  return -2;
}

}  // namespace klein
