// attn_tc.cu — causal softmax attention for prefill on the tcgen05 tensor cores
// (LMDrive page §2.3 LlamaAttention; "LLM 核心机制交互讲义" §02.1 causal mask):
//
//   O = softmax(Q K^T / sqrt(d_h) + M) V,   M_ij = 0 for key j <= query position i,
//                                            -inf otherwise,
// with GQA: query head h reads KV head h / (H / H_kv) (repeat_kv without
// materialising the repeat).
//
// One CTA per (batch, head, 128-row query tile), heaviest tiles first. Key/value
// tiles of 128 rows stream through a 2-stage TMA ring; tiles entirely above the
// diagonal are never loaded, and the mask is applied only on tiles that cross it.
//   warp 0      TMA producer (Q once, then K_j and V_j per tile)
//   warp 1      TMEM allocation + single-thread MMA issue:
//                 S_j = Q K_j^T into one of two TMEM score buffers (128 columns each),
//                 O  += P_j V_j  into a TMEM accumulator (V read MN-major)
//   warps 2..5  softmax: each thread owns one query row: reads its S row from
//               TMEM, online max/sum in fp32 (base-2 exponent with log2(e)/sqrt(d_h)
//               folded into the scale), rescales O in TMEM when the max moves,
//               writes P (bf16) into shared memory in the MMA's swizzled K-major
//               layout; finally O / l is written to o[b][t][h][:].
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

constexpr int kAttnTcThreads = 192;

template <int DH>
struct AttnCfg {
  static constexpr int BQ = 128, BKV = 128;
  static constexpr int PANELS = DH / 64;      // 64-column, 128-byte swizzled panels
  static constexpr int PANEL_BYTES = 128 * 128;  // one panel of a 128-row tile
  static constexpr int Q_BYTES = BQ * DH * 2;
  static constexpr int KV_BYTES = BKV * DH * 2;
  static constexpr int P_BYTES = BQ * BKV * 2;
  static constexpr int SMEM = Q_BYTES + 4 * KV_BYTES + P_BYTES + 256 + 1024;
  static constexpr int TMEM_COLS = 512;  // S0 [0,128), S1 [128,256), O [256, 256+DH)
};

template <int DH>
__global__ void __launch_bounds__(kAttnTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ out, int B, int Tq,
                   int Tk, int H, int Hkv, float scale_log2, int* err) {
  using C = AttnCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::Q_BYTES;          // 2 stages
  uint8_t* sV = sK + 2 * C::KV_BYTES;     // 2 stages
  uint8_t* sP = sV + 2 * C::KV_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + C::P_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* v_full = bars + 3;    // [2]
  uint64_t* kv_empty = bars + 5;  // [2]
  uint64_t* s_full = bars + 7;    // [2]
  uint64_t* p_full = bars + 9;
  uint64_t* o_full = bars + 10;
  uint64_t* drain = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nq = (Tq + C::BQ - 1) / C::BQ;
  const int lin = blockIdx.x;
  const int qt = nq - 1 - lin / (B * H);  // heaviest query tiles first
  const int bh = lin % (B * H);
  const int h = bh % H, b = bh / H;
  const int hk = h / (H / Hkv);
  const int q0 = qt * C::BQ;
  const int off = Tk - Tq;  // query row i sits at position off + i
  const int last_key = min(off + q0 + C::BQ - 1, Tk - 1);
  const int n_kv = last_key / C::BKV + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
    }
    mbar_init(p_full, 4);  // one arrival per softmax warp
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
      for (int p = 0; p < C::PANELS; ++p)
        tma_load_3d(sQ + p * C::PANEL_BYTES, &tmQ, q_full, p * 64, q0, b * H + h);
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&kv_empty[st], ((j >> 1) & 1) ^ 1, err, 0x21)) break;
        mbar_arrive_expect_tx(&k_full[st], C::KV_BYTES);
        for (int p = 0; p < C::PANELS; ++p)
          tma_load_3d(sK + st * C::KV_BYTES + p * C::PANEL_BYTES, &tmK, &k_full[st], p * 64,
                      j * C::BKV, b * Hkv + hk);
        mbar_arrive_expect_tx(&v_full[st], C::KV_BYTES);
        for (int p = 0; p < C::PANELS; ++p)
          tma_load_3d(sV + st * C::KV_BYTES + p * C::PANEL_BYTES, &tmV, &v_full[st], p * 64,
                      j * C::BKV, b * Hkv + hk);
        issued = j + 1;
      }
      pdl_trigger();
      // every issued load must land before the CTA may exit
      mbar_wait(q_full, 0, err, 0x22);
      for (int j = max(0, issued - 2); j < issued; ++j) {
        mbar_wait(&k_full[j & 1], (j >> 1) & 1, err, 0x22);
        mbar_wait(&v_full[j & 1], (j >> 1) & 1, err, 0x22);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_o = umma_idesc_bf16(128, DH, 0, 1);  // V is MN-major
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0, err, 0x23);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&k_full[st], (j >> 1) & 1, err, 0x24)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t o = (kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32;
          umma_bf16(tmem_base + st * 128, umma_desc_sw128(q_addr + o, 16, 1024),
                    umma_desc_sw128(k_addr + o, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 1 < n_kv && !issue_s(j + 1)) break;
        if (!mbar_wait(p_full, j & 1, err, 0x25)) break;
        const int st = j & 1;
        if (!mbar_wait(&v_full[st], (j >> 1) & 1, err, 0x26)) break;
        tc_fence_after();
        const uint32_t p_addr = smem_u32(sP);
        const uint32_t v_addr = smem_u32(sV + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::BKV / 16; ++kk) {
          const uint64_t ad =
              umma_desc_sw128(p_addr + (kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32, 16, 1024);
          // MN-major V: 16 keys = 16 rows of 128 B; the next 64 head dims are one
          // panel (128 rows x 128 B) further.
          const uint64_t bd = umma_desc_sw128(v_addr + kk * 16 * 128, C::PANEL_BYTES, 1024);
          umma_bf16(tmem_base + 256, ad, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&kv_empty[st]);
        umma_commit(o_full);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, err, 0x27);
    }
  } else {
    // ---------------- softmax / correction / output (warps 2..5)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const int qp = off + q0 + r;        // its position
    const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t t_o = t_row + 256;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j & 1;
      if (!mbar_wait(&s_full[st], (j >> 1) & 1, err, 0x28)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(t_row + st * 128 + c * 32, s[c]);
      tmem_wait_ld();
      const bool need_mask = j * C::BKV + C::BKV - 1 > off + q0;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float v = s[c][i] * scale_log2;
          if (need_mask && j * C::BKV + c * 32 + i > qp) v = -INFINITY;
          s[c][i] = v;
          mx = fmaxf(mx, v);
        }
      const float m_new = fmaxf(m_run, mx);
      const float alpha = ex2_approx(m_run - m_new);  // 0 on the first tile
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p = ex2_approx(s[c][i] - m_new);
          s[c][i] = p;
          rs += p;
        }
      l_run = l_run * alpha + rs;
      m_run = m_new;
      if (j > 0) {
        // P_{j-1} V_{j-1} must be complete: O is stable and the P buffer is free.
        if (!mbar_wait(o_full, (j - 1) & 1, err, 0x29)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < DH / 32; ++c) {
            float o[32];
            tmem_ld32(t_o + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(t_o + c * 32, o);
          }
          tmem_wait_st();
        }
      }
      // P row r into the swizzled K-major layout: key c -> panel c/64, 16-byte
      // chunk (c%64)/8 stored at chunk ^ (r % 8).
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int c = ch >> 2, i0 = (ch & 3) * 8;
        uint4 pk;
        pk.x = pack_bf16x2(s[c][i0 + 0], s[c][i0 + 1]);
        pk.y = pack_bf16x2(s[c][i0 + 2], s[c][i0 + 3]);
        pk.z = pack_bf16x2(s[c][i0 + 4], s[c][i0 + 5]);
        pk.w = pack_bf16x2(s[c][i0 + 6], s[c][i0 + 7]);
        const int panel = ch >> 3, c16 = ch & 7;
        *reinterpret_cast<uint4*>(sP + panel * C::PANEL_BYTES + r * 128 + ((c16 ^ (r & 7)) << 4)) =
            pk;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && mbar_wait(o_full, (n_kv - 1) & 1, err, 0x2a)) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const bool store = q0 + r < Tq;
      bf16* dst = out + (((long long)b * Tq + q0 + r) * H + h) * DH;
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        float o[32];
        tmem_ld32(t_o + c * 32, o);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float t[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) t[i] = o[q * 8 + i] * inv_l;
            store8(dst + c * 32 + q * 8, t);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int DH>
static cudaError_t run_attn(const void* q, const void* k, const void* v, void* o, int B, int Tq,
                            int Tk, int H, int Hkv, int k_stride, int* err, cudaStream_t s) {
  using C = AttnCfg<DH>;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_3d_bf16(&tq, q, (uint64_t)B * H, Tq, DH, (uint64_t)Tq * DH, 128) ||
      !make_tmap_3d_bf16(&tk, k, (uint64_t)B * Hkv, Tk, DH, (uint64_t)k_stride * DH, 128) ||
      !make_tmap_3d_bf16(&tv, v, (uint64_t)B * Hkv, Tk, DH, (uint64_t)k_stride * DH, 128))
    return cudaErrorInvalidValue;
  auto kern = attn_tc_kernel<DH>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int nq = (Tq + 127) / 128;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  return launch_k(kern, nq * B * H, kAttnTcThreads, C::SMEM, s, tq, tk, tv, (bf16*)o, B, Tq, Tk, H,
                  Hkv, scale_log2, err);
}

cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* o, int B, int Tq,
                           int Tk, int H, int Hkv, int dh, int k_stride, int* err,
                           cudaStream_t s) {
  if (B <= 0 || Tq <= 0) return cudaSuccess;
  if (dh == 128) return run_attn<128>(q, k, v, o, B, Tq, Tk, H, Hkv, k_stride, err, s);
  if (dh == 64) return run_attn<64>(q, k, v, o, B, Tq, Tk, H, Hkv, k_stride, err, s);
  return cudaErrorInvalidValue;
}

}  // namespace lb
