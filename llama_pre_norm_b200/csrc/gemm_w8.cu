// gemm_w8.cu — decode GEMMs with weight-only INT8 weights ("深入解析Llama MLP模块：SwiGLU
// 激活函数与参数配置详解" §6.4: INT8 weights cut the inference memory of the MLP; the
// decode step of "LLM 核心机制交互讲义" chapter 04 streams every weight once per token,
// so halving the weight bytes halves that part of the step).
//
// Scheme (per output row n of each nn.Linear weight): s_n = max_k |w_nk| / 127,
// q_nk = rint(w_nk / s_n) in [-127, 127], w_nk ~ s_n q_nk; decided in fp32.
//
// The GEMM is the swap-AB decode GEMM of gemm_tc.cu (weights are the 128-row
// operand, the B <= 32 tokens the N side, split-K partials) with one more stage:
//   warp 0      TMA: the INT8 weight tile (128 x 64 bytes) and the bf16 token tile
//   warps 6..9  convert the INT8 tile to bf16 (exact: |q| <= 127) into the MMA's
//               128-byte-swizzled K-major layout, one weight row per thread
//   warp 1      tcgen05.mma (M=128, N=32) on the converted tile
//   warps 2..5  epilogue: partial[split][token][n] = s_n * acc
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

constexpr int kW8Threads = 320;

// ---------------------------------------------------------------- quantization
// One CTA per row: amax in fp32, s = amax / 127 (IEEE division), q = rint(w / s).
__global__ void __launch_bounds__(256) quantize_rows_int8_kernel(const bf16* __restrict__ w,
                                                                 int8_t* __restrict__ q,
                                                                 float* __restrict__ scale, int cols) {
  __shared__ float red[32];
  pdl_wait();
  const long long row = blockIdx.x;
  const bf16* src = w + row * cols;
  float amax = 0.f;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) amax = fmaxf(amax, fabsf(__bfloat162float(src[c])));
  amax = block_max(amax, red);
  const float s = amax / 127.0f;
  if (threadIdx.x == 0) scale[row] = s;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) {
    float v = 0.f;
    if (s > 0.f) v = fminf(fmaxf(rintf(__bfloat162float(src[c]) / s), -127.f), 127.f);
    q[row * cols + c] = (int8_t)(int)v;
  }
}

cudaError_t launch_quantize_rows_int8(const void* w, void* q, float* scale, int rows, int cols,
                                      cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  return launch_k(quantize_rows_int8_kernel, rows, 256, 0, s, (const bf16*)w, (int8_t*)q, scale,
                  cols);
}

// ---------------------------------------------------------------- GEMM
template <int BN>
struct W8Cfg {
  static constexpr int STAGES = 6;
  static constexpr int RAW_BYTES = 128 * 64;      // INT8 weight tile
  static constexpr int B_BYTES = BN * 64 * 2;     // bf16 token tile
  static constexpr int CVT_BYTES = 128 * 64 * 2;  // converted bf16 weight tile
  static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
  static constexpr int SMEM = STAGES * (RAW_BYTES + B_BYTES + CVT_BYTES) + 256 + 1024;
};

template <int BN>
__global__ void __launch_bounds__(kW8Threads, 1)
    gemm_w8_kernel(const __grid_constant__ CUtensorMap tmA8, const __grid_constant__ CUtensorMap tmB,
                   const float* __restrict__ row_scale, int M, int N, int K, int kb_per, int n_split,
                   GemmEpi epi) {
  using C = W8Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sCvt = smem;                                   // STAGES x 16 KB (1024-aligned)
  uint8_t* sB = sCvt + C::STAGES * C::CVT_BYTES;          // STAGES x BN*128 B
  uint8_t* sRaw = sB + C::STAGES * C::B_BYTES;            // STAGES x 8 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRaw + C::STAGES * C::RAW_BYTES);
  uint64_t* full = bars;                      // TMA landed (raw + B)
  uint64_t* empty = bars + C::STAGES;         // raw converted and B consumed
  uint64_t* cvt_full = bars + 2 * C::STAGES;  // converted tile ready
  uint64_t* cvt_empty = bars + 3 * C::STAGES; // converted tile consumed by the MMA
  uint64_t* tfull = bars + 4 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 5);  // one MMA commit + four converter warps
      mbar_init(&cvt_full[s], 4);
      mbar_init(&cvt_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tmA8);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  const int num_m = (M + 127) / 128, num_n = (N + BN - 1) / BN;
  const int KB = (K + 63) / 64;
  const int units = num_m * num_n * n_split;
  auto decode = [&](int u, int& mt, int& nt, int& sp, int& kb0, int& kb1) {
    const int mn = num_m * num_n;
    sp = u / mn;
    const int rem = u - sp * mn;
    mt = rem % num_m;
    nt = rem / num_m;
    kb0 = sp * kb_per;
    kb1 = min(KB, kb0 + kb_per);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      uint32_t stage = 0, phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mt, nt, sp, kb0, kb1;
        decode(u, mt, nt, sp, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, epi.err, 0x41)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::RAW_BYTES + C::B_BYTES);
          tma_load_2d(sRaw + stage * C::RAW_BYTES, &tmA8, &full[stage], kb * 64, mt * 128);
          tma_load_2d(sB + stage * C::B_BYTES, &tmB, &full[stage], kb * 64, nt * BN);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      pdl_trigger();
      const long long first = issued > C::STAGES ? issued - C::STAGES : 0;
      for (long long i = first; i < issued; ++i)
        mbar_wait(&empty[i % C::STAGES], (uint32_t)((i / C::STAGES) & 1), epi.err, 0x42);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc = umma_idesc_bf16(128, BN, 0, 0);
      uint32_t stage = 0, phase = 0;
      int t = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++t) {
        int mt, nt, sp, kb0, kb1;
        decode(u, mt, nt, sp, kb0, kb1);
        const int acc = t & 1;
        if (!mbar_wait(&tempty[acc], ((t >> 1) & 1) ^ 1, epi.err, 0x43)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, epi.err, 0x44) ||
              !mbar_wait(&cvt_full[stage], phase, epi.err, 0x45)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sCvt + stage * C::CVT_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(d_tmem, umma_desc_sw128(a0 + k * 32, 16, 1024),
                      umma_desc_sw128(b0 + k * 32, 16, 1024), idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[stage]);
          umma_commit(&cvt_empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, epi.err, 0x46);
    }
  } else if (warp >= 6) {
    // ---------------- INT8 -> bf16 converters: thread r converts weight row r
    const int r = threadIdx.x - 6 * 32;
    // Order of the four 16-byte reads of a row. A 16-byte access is served per 8
    // threads (rows r0..r0+7): reads land on 16-byte bank group 4*(r&1) + i, writes of
    // output chunk c = 2i + h on group c ^ (r&7). Taking i = g(r>>1 & 3) ^ ii with g
    // multiplication by a generator of GF(4) ({0,1,2,3} -> {0,2,3,1}) makes both g(x)
    // and g(x) ^ x permutations, so each 8-thread phase hits 8 distinct groups on
    // both the read and the write side.
    const int rot = (0x78 >> (2 * ((r >> 1) & 3))) & 3;
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int mt, nt, sp, kb0, kb1;
      decode(u, mt, nt, sp, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_warp(&full[stage], phase, epi.err, 0x47) ||
            !mbar_wait_warp(&cvt_empty[stage], phase ^ 1, epi.err, 0x48)) {
          ok = false;
          break;
        }
        const uint8_t* src = sRaw + stage * C::RAW_BYTES + r * 64;
        uint8_t* dst = sCvt + stage * C::CVT_BYTES + r * 128;
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
          const int i = ii ^ rot;  // 16 int8 = bf16 chunks 2i and 2i+1
          const uint4 raw = *reinterpret_cast<const uint4*>(src + i * 16);
          const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t pk[8];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            // little-endian: byte j of the word is element 4w + j; sign-extend each
            const uint32_t u = wds[w];
            const float f0 = (float)((int32_t)(u << 24) >> 24), f1 = (float)((int32_t)(u << 16) >> 24);
            const float f2 = (float)((int32_t)(u << 8) >> 24), f3 = (float)((int32_t)u >> 24);
            pk[2 * w] = pack_bf16x2(f0, f1);
            pk[2 * w + 1] = pack_bf16x2(f2, f3);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = 2 * i + h;  // 16-byte chunk of the 128-byte row
            *reinterpret_cast<uint4*>(dst + ((c ^ (r & 7)) << 4)) =
                make_uint4(pk[4 * h], pk[4 * h + 1], pk[4 * h + 2], pk[4 * h + 3]);
          }
        }
        fence_proxy_async_smem();  // generic-proxy writes -> tensor core reads
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&cvt_full[stage]);
          mbar_arrive(&empty[stage]);
        }
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5): row-scaled split-K partials
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    int t = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++t) {
      int mt, nt, sp, kb0, kb1;
      decode(u, mt, nt, sp, kb0, kb1);
      const int acc = t & 1;
      if (!mbar_wait_warp(&tfull[acc], (t >> 1) & 1, epi.err, 0x49)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      const int row = mt * 128 + row_in_tile;
      const float sc = row < M ? row_scale[row] : 0.f;
      float* part = reinterpret_cast<float*>(epi.out) + (long long)sp * epi.split_stride;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tb + c * 32, v);
        tmem_wait_ld();
        if (row < M) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int tok = nt * BN + c * 32 + i;
            if (tok < N) part[(long long)tok * epi.ldo + row] = v[i] * sc;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

cudaError_t launch_gemm_w8(const void* A8, const float* row_scale, const void* B, int M, int N,
                           int K, int n_split, const GemmEpi& epi, int num_sms, cudaStream_t s) {
  if (M <= 0 || N <= 0 || K <= 0) return cudaSuccess;
  if (N > 32 || K % 64 != 0) return cudaErrorInvalidValue;
  constexpr int BN = 32;
  using C = W8Cfg<BN>;
  CUtensorMap ta, tb;
  if (!make_tmap_2d_u8(&ta, A8, (uint64_t)M, (uint64_t)K, 128, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_2d_bf16(&tb, B, (uint64_t)N, (uint64_t)K, BN)) return cudaErrorInvalidValue;
  const int KB = K / 64;
  n_split = gemm_effective_split(K, n_split);
  const int kb_per = (KB + n_split - 1) / n_split;
  const long long units = (long long)((M + 127) / 128) * n_split;
  const int grid = (int)std::min<long long>(units, num_sms);
  auto kern = gemm_w8_kernel<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_k(kern, grid, kW8Threads, C::SMEM, s, ta, tb, row_scale, M, N, K, kb_per, n_split,
                  epi);
}

}  // namespace lb
