// tcgen05 flash attention for the Klein block: O = softmax(Q K^T / sqrt(128)) V
// per (batch item, head), over every row of the sequence view, no mask
// (Diffusers release blog for FLUX.3 Klein, "Speed, architecture, and how the
// tokens move": in the joint stage every token attends to every token, text
// padding included; in stage 1 each stream attends to itself, which the
// caller expresses as a view over that stream's rows).
//
// One CTA = two 128-row query tiles (a, b) of one head, sharing every K/V
// tile. Roles (320 threads):
//   warp 0      TMA: both Q tiles once, then K and V^T tiles of 128 keys
//               through a 2-stage ring
//   warp 1      TMEM allocator and MMA issuer. Per key tile j, for each query
//               tile t in turn: O_t += P_t V_j (P_t read from tensor memory),
//               then S_t = Q_t K_{j+1}^T. While one tile's softmax runs, the
//               tensor core works on the other tile.
//   warps 2..5  softmax of tile a, warps 6..9 softmax of tile b: one query
//               row per thread, scores read from TMEM, running max / sum in the
//               exp2 domain, P written back over the scores in TMEM as bf16.
//               The running max is only moved (and the TMEM output rescaled)
//               when a row's max grows by more than 2^8, so rescales are rare;
//               the bound keeps P <= 256. Final 1/l normalisation and bf16
//               store into the out-projection's A operand.
// Tensor memory (512 columns): tile t owns S_t (128 fp32 columns, P_t in its
// first 64 as packed bf16) and O_t (128 fp32 columns). P stays in tensor
// memory: written to shared memory instead, its stores and the MMA's reads of
// it add about 96 KB of shared-memory traffic per key tile on top of the
// operands, more than the shared-memory bandwidth leaves room for.
// Keys past the end of the view are zero-filled by TMA and masked to -inf.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace klein {

namespace {
constexpr int kTileBytes = 128 * 128 * 2;  // a 128 x 128 bf16 tile = 2 swizzle chunks of 16 KB
constexpr int kOffQ = 0;                   // 2 query tiles
constexpr int kOffK = 2 * kTileBytes;      // 2 stages
constexpr int kOffV = 4 * kTileBytes;      // 2 stages
constexpr int kOffBar = 6 * kTileBytes;
constexpr int kSmem = kOffBar + 256 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 320;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale only when the max grows by > 2^8
}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_vt, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* kv_empty = bars + 5;  // [2]
  uint64_t* s_full = bars + 7;    // [2 tiles]: scores ready (phase j), final output ready (phase nkv)
  uint64_t* p_full = bars + 9;    // [2 tiles][2 halves of the keys]
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * a.heads + head;
  const int q_row0 = blockIdx.x * 256;
  const int nkv = (a.rows + 127) / 128;

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[2 * s], 128);
      mbar_init(&p_full[2 * s + 1], 128);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&map_q);
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_vt);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
  pdl_trigger();
  pdl_wait();  // q, k, v^T and the output are touched only after the previous kernel completes

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * kTileBytes);
      for (int t = 0; t < 2; ++t) {
        tma_load_3d(smem + kOffQ + t * kTileBytes, &map_q, q_full, 0, q_row0 + 128 * t, bh);
        tma_load_3d(smem + kOffQ + t * kTileBytes + kTileBytes / 2, &map_q, q_full, 64, q_row0 + 128 * t, bh);
      }
      StageLog klog, vlog;
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&kv_empty[st], ((j >> 1) & 1) ^ 1, 0x201)) break;
        uint8_t* kd = smem + kOffK + st * kTileBytes;
        uint8_t* vd = smem + kOffV + st * kTileBytes;
        mbar_arrive_expect_tx(&k_full[st], kTileBytes);
        klog.armed(st, (j >> 1) & 1);
        tma_load_3d(kd, &map_k, &k_full[st], 0, j * 128, bh);
        tma_load_3d(kd + kTileBytes / 2, &map_k, &k_full[st], 64, j * 128, bh);
        mbar_arrive_expect_tx(&v_full[st], kTileBytes);
        vlog.armed(st, (j >> 1) & 1);
        tma_load_3d(vd, &map_vt, &v_full[st], j * 128, 0, bh);
        tma_load_3d(vd + kTileBytes / 2, &map_vt, &v_full[st], j * 128 + 64, 0, bh);
      }
      // no TMA write may land in shared memory after the CTA exits
      if (mbar_wait(q_full, 0, 0x209)) {
        klog.drain(k_full, 2, 0x209);
        vlog.drain(v_full, 2, 0x209);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      auto issue_s = [&](int t, int j) {
        const uint32_t q0 = smem_u32(smem + kOffQ + t * kTileBytes);
        const uint32_t k0 = smem_u32(smem + kOffK + (j & 1) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
          umma_bf16(tmem_base + t * 256, sw128_desc(q0 + off), sw128_desc(k0 + off), idesc, kk != 0);
        }
        umma_commit(&s_full[t]);
      };
      bool ok = mbar_wait(q_full, 0, 0x202) && mbar_wait(&k_full[0], 0, 0x203);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int st = j & 1;
        for (int t = 0; t < 2 && ok; ++t) {
          if (t == 0 && !mbar_wait(&v_full[st], (j >> 1) & 1, 0x205)) { ok = false; break; }
          const uint32_t v0 = smem_u32(smem + kOffV + st * kTileBytes);
          for (int half = 0; half < 2; ++half) {
            if (!mbar_wait(&p_full[2 * t + half], j & 1, 0x204)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk = 4 * half; kk < 4 * half + 4; ++kk) {
              const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
              umma_bf16_tmem_a(tmem_base + t * 256 + 128, tmem_base + t * 256 + kk * 8, sw128_desc(v0 + off),
                               idesc, (j | kk) != 0);
            }
          }
          if (!ok) break;
          if (t == 1) umma_commit(&kv_empty[st]);
          if (j + 1 < nkv) {
            if (t == 0) {
              if (!mbar_wait(&k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, 0x206)) { ok = false; break; }
              tc_fence_after();
            }
            issue_s(t, j + 1);
          } else {
            umma_commit(&s_full[t]);  // output of tile t final
          }
        }
      }
      // every MMA issued here has completed before TMEM is freed
      umma_commit(drain);
      mbar_wait(drain, 0, 0x20a);
    }
  } else {
    const int t = (warp - 2) >> 2;         // query tile of this warpgroup
    const int quarter = warp & 3;          // TMEM lane quarter of this warp
    const int rloc = quarter * 32 + lane;
    const int q_row = q_row0 + 128 * t + rloc;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t s_col = lane_base + t * 256;
    const uint32_t o_col = s_col + 128;
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;
    float s[128];
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait(&s_full[t], j & 1, 0x207)) { ok = false; break; }
      tc_fence_after();
      tmem_ld128(s_col, s);
      const int lim = a.rows - j * 128;  // valid keys in this tile
      const bool tail = lim < 128;
      if (tail) {
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = (i < lim) ? s[i] : -INFINITY;
      }
      // row max: 8 independent chains of three-input maxima
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = fmax3(s[q], s[q + 8], s[q + 16]);
#pragma unroll
      for (int i = 24; i < 120; i += 16) {
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = fmax3(m8[q], s[i + q], s[i + 8 + q]);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = fmaxf(m8[q], s[120 + q]);
      const float mx = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], fmax3(m8[5], m8[6], m8[7])));
      const float m_cand = mx * sl2;
      // move the running max only if it grows past the threshold
      const bool grow = m_cand > m_run + kRescaleThreshold;
      const float m_new = grow ? m_cand : m_run;
      const float alpha = fast_exp2(m_run - m_new);
      // p = exp2(s * scale - m): the affine step two lanes per instruction,
      // exp2 on MUFU, sums two-wide in four independent accumulators. P goes
      // back to TMEM in two halves of 64 keys, each released to the MMA warp
      // on its own barrier, so O += P V over the first half runs while the
      // second half is being exponentiated.
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int i = 64 * half; i < 64 * half + 64; i += 2) {  // masked keys: exp2(-inf) = 0 exactly
          float x0, x1;
          ffma2(x0, x1, s[i], s[i + 1], sl2, sl2, -m_new, -m_new);
          const float p0 = fast_exp2(x0);
          const float p1 = fast_exp2(x1);
          fadd2(sa[(i >> 1) & 3], sb[(i >> 1) & 3], p0, p1);
          pk[(i >> 1) & 31] = pack_bf16(p0, p1);
        }
        // the output row is rescaled (rarely) before any P V of this key
        // tile is released, and after half the scores are consumed
        if (half == 0 && j > 0 && __any_sync(0xffffffffu, grow)) {
          float o[32];
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            tmem_ld32(o_col + 32 * c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(o_col + 32 * c, o);
          }
        }
        tmem_st32(s_col + 32 * half, reinterpret_cast<const float*>(pk));
        tc_fence_before();
        mbar_arrive(&p_full[2 * t + half]);
      }
      float sum4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) sum4[q] = sa[q] + sb[q];
      l_run = l_run * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
      m_run = m_new;
    }
    if (ok && mbar_wait(&s_full[t], nkv & 1, 0x208)) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      __nv_bfloat16* dst = a.out + ((long long)b * a.rows + q_row) * a.out_ld + head * kHeadDim;
      float o[32];
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(o_col + 32 * c, o);
        if (q_row < a.rows) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            *reinterpret_cast<uint4*>(dst + 32 * c + i) =
                make_uint4(pack_bf16(o[i] * inv, o[i + 1] * inv), pack_bf16(o[i + 2] * inv, o[i + 3] * inv),
                           pack_bf16(o[i + 4] * inv, o[i + 5] * inv), pack_bf16(o[i + 6] * inv, o[i + 7] * inv));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

int launch_attention(const AttnArgs& a, cudaStream_t s) {
  static bool configured[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return -1;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
      return -1;
    configured[dev] = true;
  }
  if (a.rows <= 0 || a.batch <= 0) return 0;
  CUtensorMap mq, mk, mvt;
  const uint64_t bh = (uint64_t)a.batch * a.heads, rp = a.rows_pad;
  if (make_map_3d(&mq, a.q, kHeadDim, a.rows, bh, kHeadDim * 2, rp * kHeadDim * 2, 64, 128) ||
      make_map_3d(&mk, a.k, kHeadDim, a.rows, bh, kHeadDim * 2, rp * kHeadDim * 2, 64, 128) ||
      make_map_3d(&mvt, a.vt, a.rows, kHeadDim, bh, rp * 2, rp * kHeadDim * 2, 64, 128))
    return -2;
  const cudaError_t e = launch_kernel(attn_kernel, dim3((a.rows + 255) / 256, a.heads, a.batch), dim3(kThreads), kSmem,
                                      s, 1, mq, mk, mvt, a);
  note_launch();
  return (e == cudaSuccess && cudaPeekAtLastError() == cudaSuccess) ? 0 : -1;
}



}  // namespace klein
