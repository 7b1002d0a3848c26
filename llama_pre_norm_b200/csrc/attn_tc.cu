// attn_tc.cu — causal softmax attention for prefill on the tcgen05 tensor cores
// (LMDrive page §2.3 LlamaAttention; "LLM 核心机制交互讲义" §02.1 causal mask):
//
//   O = softmax(Q K^T / sqrt(d_h) + M) V,   M_ij = 0 for key j <= query position i,
//                                            -inf otherwise,
// with GQA: query head h reads KV head h / (H / H_kv) (repeat_kv without
// materialising the repeat).
//
// One CTA per (batch, head, pair of 128-row query tiles A and B), heaviest pairs
// first. Both tiles consume the same 128-key K/V tiles, which stream through a
// 2-stage TMA ring; K/V tiles above the diagonal are never loaded and the mask is
// applied only on tiles that cross it.
//   warp 0       TMA producer (Q_A, Q_B once; then K_j, V_j)
//   warp 1       TMEM allocation + single-thread MMA issue, interleaving the tiles:
//                  PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), ...
//                S_t = Q_t K_j^T lands in tile t's 128 score columns; the softmax
//                writes P_t (bf16) over the first 64 of those columns and
//                O_t += P_t V_j reads P_t straight from TMEM (V MN-major in smem).
//                S_t(j+1) overwrites P_t(j); it is issued right behind PV_t(j), which
//                is safe because tcgen05.mma operations of one thread execute (and
//                complete) in issue order. (Waiting for PV_t(j) to complete first
//                measured 3% slower.)
//   warps 2..5   softmax of tile A, warps 6..9 softmax of tile B: one query row per
//                thread (= TMEM lane); online max/sum in fp32 with log2(e)/sqrt(d_h)
//                folded into the exponent's FMA and a three-input max over eight
//                independent chains (measured:
//                packed f32x2 forms and an FMA-pipe polynomial for part of the
//                exponentials were slower here). The running max is only
//                moved (and O rescaled in TMEM) when a row's max grows by more than
//                2^8, so most tiles skip the rescale; P <= 2^8 stays exact enough in
//                bf16 and the final O / l uses the same reference max.
// While one tile's softmax runs, the tensor core works on the other tile.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

constexpr int kAttnTcThreads = 320;
constexpr float kRescaleLog2 = 8.0f;

// ---------------------------------------------------------------- softmax arithmetic
// Three-input max (sm_100): one instruction per two new scores.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int DH>
struct AttnCfg {
  static constexpr int BQ = 128, BKV = 128;
  static constexpr int PANELS = DH / 64;         // 64-column, 128-byte swizzled panels
  static constexpr int PANEL_BYTES = 128 * 128;  // one panel of a 128-row tile
  static constexpr int Q_BYTES = BQ * DH * 2;
  static constexpr int KV_BYTES = BKV * DH * 2;
  static constexpr int SMEM = 2 * Q_BYTES + 4 * KV_BYTES + 256 + 1024;
  static constexpr int TMEM_COLS = 512;  // S/P of tile t at 128 t, O of tile t at 256 + 128 t
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
  uint8_t* sQ = smem;                      // tile A, then tile B
  uint8_t* sK = sQ + 2 * C::Q_BYTES;       // 2 stages
  uint8_t* sV = sK + 2 * C::KV_BYTES;      // 2 stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + 2 * C::KV_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;    // [2 stages]
  uint64_t* v_full = bars + 3;    // [2 stages]
  uint64_t* kv_empty = bars + 5;  // [2 stages]
  uint64_t* s_full = bars + 7;    // [2 tiles]
  uint64_t* p_full = bars + 9;    // [2 tiles]
  uint64_t* o_full = bars + 11;   // [2 tiles]
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int npairs = (Tq + 2 * C::BQ - 1) / (2 * C::BQ);
  const int lin = blockIdx.x;
  const int pr = npairs - 1 - lin / (B * H);  // heaviest pairs first
  const int bh = lin % (B * H);
  const int h = bh % H, b = bh / H;
  const int hk = h / (H / Hkv);
  const int q0 = pr * 2 * C::BQ;
  const int off = Tk - Tq;  // query row i sits at position off + i
  const bool hasB = q0 + C::BQ < Tq;
  int n_t[2];
  n_t[0] = min(off + q0 + C::BQ - 1, Tk - 1) / C::BKV + 1;
  n_t[1] = hasB ? min(off + q0 + 2 * C::BQ - 1, Tk - 1) / C::BKV + 1 : 0;
  const int n_max = max(n_t[0], n_t[1]);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);  // one arrival per softmax warp of the tile
      mbar_init(&o_full[i], 1);
    }
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
      mbar_arrive_expect_tx(q_full, (hasB ? 2 : 1) * C::Q_BYTES);
      for (int t = 0; t < (hasB ? 2 : 1); ++t)
        for (int p = 0; p < C::PANELS; ++p)
          tma_load_3d(sQ + t * C::Q_BYTES + p * C::PANEL_BYTES, &tmQ, q_full, p * 64,
                      q0 + t * C::BQ, b * H + h);
      int issued = 0;
      for (int j = 0; j < n_max; ++j) {
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
      auto issue_s = [&](int t, int st) {
        const uint32_t q_addr = smem_u32(sQ + t * C::Q_BYTES);
        const uint32_t k_addr = smem_u32(sK + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t o = (kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32;
          umma_bf16(tmem_base + t * 128, umma_desc_sw128(q_addr + o, 16, 1024),
                    umma_desc_sw128(k_addr + o, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, int st, int j) {
        const uint32_t v_addr = smem_u32(sV + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::BKV / 16; ++kk) {
          // P_t: 8 TMEM columns per 16 keys. V: 16 keys = 16 rows of 128 B; the next
          // 64 head dims are one panel (128 rows x 128 B) further.
          const uint64_t bd = umma_desc_sw128(v_addr + kk * 16 * 128, C::PANEL_BYTES, 1024);
          umma_bf16_tmem_a(tmem_base + 256 + t * 128, tmem_base + t * 128 + kk * 8, bd, idesc_o,
                           (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&o_full[t]);
      };
      bool ok = mbar_wait(q_full, 0, err, 0x23) && mbar_wait(&k_full[0], 0, err, 0x24);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          if (n_t[t] > 0) issue_s(t, 0);
      }
      // Per tile: PV_t(j), then (once PV_t(j) has completed) S_t(j+1). Tile A's
      // softmax of j+1 then overlaps tile B's PV(j) and S(j+1), and vice versa.
      for (int j = 0; j < n_max && ok; ++j) {
        const int st = j & 1;
        bool v_ready = false, k_next_ready = false;
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= n_t[t]) continue;
          if (!mbar_wait(&p_full[t], j & 1, err, 0x25)) { ok = false; break; }
          if (!v_ready && !mbar_wait(&v_full[st], (j >> 1) & 1, err, 0x26)) { ok = false; break; }
          v_ready = true;
          tc_fence_after();
          issue_pv(t, st, j);
          if (j + 1 < n_t[t]) {
            if (!k_next_ready &&
                !mbar_wait(&k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, err, 0x24)) { ok = false; break; }
            k_next_ready = true;
            // S_t(j+1) overwrites P_t(j), which PV_t(j) reads: tcgen05.mma operations
            // issued by one thread execute in issue order, so it follows PV_t(j) at once.
            issue_s(t, (j + 1) & 1);
          }
        }
        if (!ok) break;
        umma_commit(&kv_empty[st]);  // K_j, V_j free once every MMA so far has completed
      }
      umma_commit(drain);
      mbar_wait(drain, 0, err, 0x28);
    }
  } else {
    // ---------------- softmax / correction / output (warps 2..5: tile A, 6..9: tile B)
    const int t = (warp - 2) >> 2;
    const int n = n_t[t];
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const int row0 = q0 + t * C::BQ;
    const int qp = off + row0 + r;      // its position
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t t_s = lane_base + t * 128;
    const uint32_t t_o = lane_base + 256 + t * 128;
    float m_ref = -INFINITY, l_run = 0.f;
    bool ok = n > 0;
    for (int j = 0; j < n && ok; ++j) {
      if (!mbar_wait_warp(&s_full[t], j & 1, err, 0x29)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool need_mask = j * C::BKV + C::BKV - 1 > off + row0;  // uniform in the CTA
      float s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, s[c]);
      tmem_wait_ld();
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (j * C::BKV + c * 32 + i > qp) s[c][i] = -INFINITY;
      }
      // row max of the raw scores (the scale is positive), three at a time in eight
      // independent chains, so that the exponentials wait for a short tree rather
      // than for 64 dependent steps
      float m8[8];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        m8[2 * c] = -INFINITY;
        m8[2 * c + 1] = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          m8[2 * c] = max3(m8[2 * c], s[c][i], s[c][i + 1]);
          m8[2 * c + 1] = max3(m8[2 * c + 1], s[c][i + 2], s[c][i + 3]);
        }
      }
      const float mxr =
          max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      const float mx = mxr * scale_log2;
      // Move the reference max only when this row's max grew by more than 2^8
      // (always on the first tile, where the reference is still -inf).
      const bool move = mx > m_ref + kRescaleLog2;
      const float m_new = move ? mx : m_ref;
      const float alpha = move ? ex2_approx(m_ref - m_new) : 1.f;  // 0 on the first tile
      // p = 2^(s * scale - m): the scale folded into one FMA per key, the row sum in two
      // independent accumulators. P is packed in place as bf16 pairs (word k of chunk c:
      // keys 32c + 2k, 32c + 2k + 1, over elements already consumed) and stored over
      // the first 64 score columns (column c: keys 2c, 2c+1); keys 32c.. land in
      // columns 16c.., whose scores are already in registers.
      const float nm = -m_new;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ex2_approx(fmaf(s[c][i], scale_log2, nm));
          const float p1 = ex2_approx(fmaf(s[c][i + 1], scale_log2, nm));
          rs0 += p0;
          rs1 += p1;
          s[c][i >> 1] = __uint_as_float(pack_bf16x2(p0, p1));
        }
        tmem_st16(t_s + c * 16, *reinterpret_cast<const uint32_t(*)[16]>(s[c]));
      }
      l_run = l_run * alpha + (rs0 + rs1);
      m_ref = m_new;
      if (j > 0 && __any_sync(0xffffffffu, move)) {
        // O_t holds PV_t(j-1) in full: S_t(j), issued after PV_t(j-1), has completed,
        // and MMAs complete in issue order. It is rescaled before this tile's P is
        // released to the MMA (PV_t(j) waits for that release).
        if (!mbar_wait_warp(&o_full[t], (j - 1) & 1, err, 0x2a)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < DH / 32; ++c) {
          float o[32];
          tmem_ld32(t_o + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(t_o + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    if (ok && mbar_wait_warp(&o_full[t], (n - 1) & 1, err, 0x2b)) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const bool store = row0 + r < Tq;
      bf16* dst = out + (((long long)b * Tq + row0 + r) * H + h) * DH;
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        float o[32];
        tmem_ld32(t_o + c * 32, o);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float tt[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) tt[i] = o[q * 8 + i] * inv_l;
            store8(dst + c * 32 + q * 8, tt);
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
  static std::atomic<unsigned long long> attr_done{0};
  if (cudaError_t e = ensure_smem_attr(kern, C::SMEM, attr_done); e != cudaSuccess)
    return e;
  const int npairs = (Tq + 255) / 256;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  return launch_k(kern, npairs * B * H, kAttnTcThreads, C::SMEM, s, tq, tk, tv, (bf16*)o, B, Tq, Tk,
                  H, Hkv, scale_log2, err);
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
