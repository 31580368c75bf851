// tcgen05 flash attention for the Klein block: O = softmax(Q K^T / sqrt(128)) V
// per (batch item, head), over every row of the sequence view, no mask
// (Diffusers release blog for FLUX.3 Klein, "Speed, architecture, and how the
// tokens move": in the joint stage every token attends to every token, text
// padding included; in stage 1 each stream attends to itself, which the
// caller expresses as a view over that stream's rows).
//
// One CTA = one 128-row query tile of one head. Roles (192 threads):
//   warp 0      TMA: Q once, then K and V^T tiles of 128 keys, 2 stages
//   warp 1      TMEM allocator and MMA issuer: S = Q K^T into one of two
//               TMEM score buffers (so S_{j+1} overlaps the softmax of S_j),
//               then O += P V into the TMEM output accumulator
//   warps 2..5  softmax: one query row per thread, online max / sum in the
//               exp2 domain, P written to shared memory as bf16 in the
//               128-byte-swizzled K-major layout the tensor core reads, the
//               TMEM output row rescaled when the running max grows; final
//               normalisation and the bf16 store into the out-projection's
//               A operand.
// Keys past the end of the view are zero-filled by TMA and masked to -inf.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace klein {

namespace {
constexpr int kTileBytes = 128 * 128 * 2;  // a 128 x 128 bf16 tile = 2 swizzle chunks of 16 KB
constexpr int kOffQ = 0;
constexpr int kOffK = kTileBytes;              // 2 stages
constexpr int kOffV = 3 * kTileBytes;          // 2 stages
constexpr int kOffP = 5 * kTileBytes;
constexpr int kOffBar = 6 * kTileBytes;
constexpr int kSmem = kOffBar + 256 + 1024;
constexpr uint32_t kTmemCols = 512;            // S0 | S1 | O | unused
constexpr uint32_t kColO = 256;
}  // namespace

__global__ void __launch_bounds__(192, 1)
    attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_vt, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* v_full = bars + 3;   // [2]
  uint64_t* kv_empty = bars + 5; // [2]
  uint64_t* s_full = bars + 7;   // [2]
  uint64_t* p_full = bars + 9;
  uint64_t* o_done = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q_tile = blockIdx.x;
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * a.heads + head;
  const int q_row0 = q_tile * 128;
  const int nkv = (a.rows + 127) / 128;

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
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

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_3d(smem + kOffQ, &map_q, q_full, 0, q_row0, bh);
      tma_load_3d(smem + kOffQ + kTileBytes / 2, &map_q, q_full, 64, q_row0, bh);
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&kv_empty[st], ((j >> 1) & 1) ^ 1, 0x201)) break;
        uint8_t* kd = smem + kOffK + st * kTileBytes;
        uint8_t* vd = smem + kOffV + st * kTileBytes;
        mbar_arrive_expect_tx(&k_full[st], kTileBytes);
        tma_load_3d(kd, &map_k, &k_full[st], 0, j * 128, bh);
        tma_load_3d(kd + kTileBytes / 2, &map_k, &k_full[st], 64, j * 128, bh);
        mbar_arrive_expect_tx(&v_full[st], kTileBytes);
        tma_load_3d(vd, &map_vt, &v_full[st], j * 128, 0, bh);
        tma_load_3d(vd + kTileBytes / 2, &map_vt, &v_full[st], j * 128 + 64, 0, bh);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t q0 = smem_u32(smem + kOffQ);
      const uint32_t p0 = smem_u32(smem + kOffP);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&k_full[st], (j >> 1) & 1, 0x202)) return false;
        tc_fence_after();
        const uint32_t k0 = smem_u32(smem + kOffK + st * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
          umma_bf16(tmem_base + st * 128, sw128_desc(q0 + off), sw128_desc(k0 + off), idesc, kk != 0);
        }
        umma_commit(&s_full[st]);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, 0x203);
      if (ok) {
        tc_fence_after();
        ok = issue_s(0);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv && !issue_s(j + 1)) break;
        if (!mbar_wait(p_full, j & 1, 0x204)) break;
        tc_fence_after();
        const int st = j & 1;
        if (!mbar_wait(&v_full[st], (j >> 1) & 1, 0x205)) break;
        tc_fence_after();
        const uint32_t v0 = smem_u32(smem + kOffV + st * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
          umma_bf16(tmem_base + kColO, sw128_desc(p0 + off), sw128_desc(v0 + off), idesc, (j | kk) != 0);
        }
        umma_commit(&kv_empty[st]);
        umma_commit(o_done);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int rloc = quarter * 32 + lane;
    const int q_row = q_row0 + rloc;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    uint8_t* prow = smem + kOffP + rloc * 128;
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;
    float s[128];
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1, 0x206)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + sb * 128 + 32 * c, s + 32 * c);
      const int lim = a.rows - j * 128;  // valid keys in this tile
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        s[i] = (i < lim) ? s[i] * sl2 : -INFINITY;
        mx = fmaxf(mx, s[i]);
      }
      const float m_new = fmaxf(m_run, mx);
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        s[i] = fast_exp2(s[i] - m_new);
        sum += s[i];
      }
      if (j > 0) {
        if (!mbar_wait(o_done, (j - 1) & 1, 0x207)) { ok = false; break; }
        tc_fence_after();
      }
      const float alpha = fast_exp2(m_run - m_new);
      if (j > 0 && __any_sync(0xffffffffu, m_new > m_run)) {
        float o[32];
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(lane_base + kColO + 32 * c, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(lane_base + kColO + 32 * c, o);
        }
      }
      l_run = l_run * alpha + sum;
      m_run = m_new;
      // P row -> two 128-byte swizzled chunks (keys 0..63, 64..127)
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int chunk = u >> 3;
        const int unit = u & 7;
        uint8_t* dst = prow + chunk * (kTileBytes / 2) + ((unit ^ (rloc & 7)) << 4);
        const float* p = s + 8 * u;
        *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16(p[0], p[1]), pack_bf16(p[2], p[3]),
                                                    pack_bf16(p[4], p[5]), pack_bf16(p[6], p[7]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && mbar_wait(o_done, (nkv - 1) & 1, 0x208)) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      __nv_bfloat16* dst = a.out + ((long long)b * a.rows + q_row) * a.out_ld + head * kHeadDim;
      float o[32];
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(lane_base + kColO + 32 * c, o);
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

int launch_attention(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mvt, const AttnArgs& a,
                     cudaStream_t s) {
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
      return -1;
    configured = true;
  }
  if (a.rows <= 0 || a.batch <= 0) return 0;
  dim3 grid((a.rows + 127) / 128, a.heads, a.batch);
  attn_kernel<<<grid, 192, kSmem, s>>>(mq, mk, mvt, a);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace klein
