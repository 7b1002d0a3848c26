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
//   warp 0      loads, per kW8K-deep K block (kW8K = 128): the INT8 weight tile (128 x
//               kW8K bytes, one contiguous bulk copy from the tile-blocked layout) and
//               the bf16 token tile (TMA), a ring whose slots also index the TMEM slots
//               of the widened tiles, so one tcgen05.commit per K block frees both
//   warps 6..17 widen the INT8 tile to bf16 (exact: |q| <= 127) straight into TMEM
//               (tcgen05.st), one weight row per thread; three groups of four warps
//               take turns over the K blocks
//   warp 1      tcgen05.mma (M=128, N=32) with the converted tile as the TMEM A operand
//   warps 2..5  epilogue: partial[split][token][n] = s_n * acc
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

// ---------------------------------------------------------------- quantization
// One CTA per row: amax in fp32, s = amax / 127 (IEEE division), q = rint(w / s).
// Codes are stored tile-blocked (w8_blocked_offset); rows of the last tile past
// `rows` are never written, so the caller zeroes the buffer first.
__global__ void __launch_bounds__(256) quantize_rows_int8_kernel(const bf16* __restrict__ w,
                                                                 int8_t* __restrict__ q,
                                                                 float* __restrict__ scale, int cols) {
  __shared__ float red[32];
  pdl_wait();
  const int row = blockIdx.x;
  const bf16* src = w + (long long)row * cols;
  float amax = 0.f;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) amax = fmaxf(amax, fabsf(__bfloat162float(src[c])));
  amax = block_max(amax, red);
  const float s = amax / 127.0f;
  if (threadIdx.x == 0) scale[row] = s;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) {
    float v = 0.f;
    if (s > 0.f) v = fminf(fmaxf(rintf(__bfloat162float(src[c]) / s), -127.f), 127.f);
    q[w8_blocked_offset(row, c, cols)] = (int8_t)(int)v;
  }
}

cudaError_t launch_quantize_rows_int8(const void* w, void* q, float* scale, int rows, int cols,
                                      cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  return launch_k(quantize_rows_int8_kernel, rows, 256, 0, s, (const bf16*)w, (int8_t*)q, scale,
                  cols);
}

// ---------------------------------------------------------------- GEMM
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}

// Four INT8 codes (bytes of u, element j in byte j) to four bf16 (two pairs, element
// order kept). Each biased byte q + 128 becomes the low byte of the fp32 pattern
// 0x4B0000xx = 2^23 + q + 128; subtracting 2^23 + 128 leaves q exactly, and since
// |q| <= 127 fits bf16's significand the bf16 is the fp32's upper half, taken by a
// byte permute. All ALU/FMA-pipe work, no int-to-float conversion instructions.
__device__ __forceinline__ void i8x4_to_bf16x4(uint32_t u, uint32_t& lo, uint32_t& hi) {
  const uint32_t x = u ^ 0x80808080u;
  constexpr float kMagic = 8388736.0f;  // 2^23 + 128
  const float f0 = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7440)) - kMagic;
  const float f1 = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7441)) - kMagic;
  const float f2 = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7442)) - kMagic;
  const float f3 = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7443)) - kMagic;
  lo = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
  hi = __byte_perm(__float_as_uint(f2), __float_as_uint(f3), 0x7632);
}

// Converter warps come in groups of four (one per TMEM lane quarter); group g widens
// the K blocks g, g + G, g + 2G, ... of the CTA's sequence, so G blocks are in flight.
constexpr int kW8ConvGroups = 3;
constexpr int kW8ConvWarps = 4 * kW8ConvGroups;
constexpr int kW8Threads = (6 + kW8ConvWarps) * 32;

template <int BN>
struct W8Cfg {
  // One pipeline step covers a kW8K-deep K block. Its ring index names both its
  // shared-memory slot (INT8 tile + token tile) and its TMEM slot (the widened tile,
  // kW8K/2 columns), so that the MMA issuer frees both with a single tcgen05.commit.
  static constexpr int HALVES = kW8K / 64;       // 64-deep pieces of a step
  static constexpr int A_COLS = kW8K / 2;        // TMEM columns of one widened tile
  static constexpr int STAGES = (512 - 2 * BN) / A_COLS < 6 ? (512 - 2 * BN) / A_COLS : 6;
  static constexpr int RAW_BYTES = 128 * kW8K;   // INT8 weight tile
  static constexpr int B_HALF = BN * 64 * 2;     // bf16 token tile, 64 K (one 128-byte swizzle atom)
  static constexpr int B_BYTES = HALVES * B_HALF;
  static constexpr int A_COL0 = 2 * BN;          // TMEM: two accumulators, then the A slots
  static constexpr int TMEM_USED = 2 * BN + STAGES * A_COLS;
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128
                                   : TMEM_USED <= 256 ? 256 : 512;
  static constexpr int SMEM = STAGES * (RAW_BYTES + B_BYTES) + 512 + 1024;
};

template <int BN>
__global__ void __launch_bounds__(kW8Threads, 1)
    gemm_w8_kernel(const uint8_t* __restrict__ A8, const __grid_constant__ CUtensorMap tmB,
                   const float* __restrict__ row_scale, int M, int N, int K, int kt_per, int n_split,
                   GemmEpi epi) {
  using C = W8Cfg<BN>;
  constexpr int RS = C::STAGES;
  static_assert(C::TMEM_USED <= 512, "TMEM");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;                           // RS x 2 x BN*128 B, 1024-aligned (128-byte swizzle)
  uint8_t* sRaw = sB + RS * C::B_BYTES;         // RS x 16 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRaw + RS * C::RAW_BYTES);
  uint64_t* full = bars;                // INT8 + token tile landed
  uint64_t* raw_free = bars + RS;       // INT8 tile read by its converter group
  uint64_t* a_full = bars + 2 * RS;     // widened tile in TMEM
  uint64_t* mma_done = bars + 3 * RS;   // the block's MMAs completed: token tile and TMEM slot free
  uint64_t* tfull = bars + 4 * RS;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&raw_free[s], 4);  // the four warps of one converter group
      mbar_init(&a_full[s], 4);
      mbar_init(&mma_done[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The INT8 weight tiles are not an input of the previous kernel: the producer
  // requests the first ones before it waits for that kernel (pdl_wait).
  if (warp != 0) pdl_wait();

  const int num_m = (M + 127) / 128, num_n = (N + BN - 1) / BN;
  const int KT = (K + kW8K - 1) / kW8K;
  const int units = num_m * num_n * n_split;
  auto decode = [&](int u, int& mt, int& nt, int& sp, int& kt0, int& kt1) {
    const int mn = num_m * num_n;
    sp = u / mn;
    const int rem = u - sp * mn;
    mt = rem % num_m;
    nt = rem / num_m;
    kt0 = sp * kt_per;
    kt1 = min(KT, kt0 + kt_per);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- loads; slot reuse needs both its INT8 tile read and its MMAs done
      int npre = 0;  // leading steps of the first unit whose INT8 tile is in flight
      if ((int)blockIdx.x < units) {
        int mt, nt, sp, kt0, kt1;
        decode(blockIdx.x, mt, nt, sp, kt0, kt1);
        npre = min(kt1 - kt0, RS);
        for (int i = 0; i < npre; ++i) {  // fresh ring: slot i is free
          mbar_arrive_expect_tx(&full[i], C::RAW_BYTES + C::B_BYTES);
          bulk_load(sRaw + i * C::RAW_BYTES, A8 + ((long long)mt * KT + kt0 + i) * C::RAW_BYTES,
                    C::RAW_BYTES, &full[i]);
        }
      }
      pdl_wait();
      uint32_t stage = 0, phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int mt, nt, sp, kt0, kt1;
        decode(u, mt, nt, sp, kt0, kt1);
        for (int kt = kt0; kt < kt1; ++kt) {
          if (issued >= npre) {
            if (!mbar_wait(&raw_free[stage], phase ^ 1, epi.err, 0x41) ||
                !mbar_wait(&mma_done[stage], phase ^ 1, epi.err, 0x4a)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], C::RAW_BYTES + C::B_BYTES);
            // one contiguous tile of the blocked layout
            bulk_load(sRaw + stage * C::RAW_BYTES, A8 + ((long long)mt * KT + kt) * C::RAW_BYTES,
                      C::RAW_BYTES, &full[stage]);
          }
          // the token tile in 64-deep pieces (past K they read as zeros)
          uint8_t* b = sB + stage * C::B_BYTES;
#pragma unroll
          for (int hh = 0; hh < C::HALVES; ++hh)
            tma_load_2d(b + hh * C::B_HALF, &tmB, &full[stage], kt * kW8K + hh * 64, nt * BN);
          ++issued;
          if (++stage == RS) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      pdl_trigger();
      const long long first = issued > RS ? issued - RS : 0;
      for (long long i = first; i < issued; ++i)
        mbar_wait(&raw_free[i % RS], (uint32_t)((i / RS) & 1), epi.err, 0x42);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: A (the widened weights) from TMEM, B from smem
      constexpr uint32_t idesc = umma_idesc_bf16(128, BN, 0, 0);
      uint32_t rs = 0, rphase = 0;
      int t = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++t) {
        int mt, nt, sp, kt0, kt1;
        decode(u, mt, nt, sp, kt0, kt1);
        const int acc = t & 1;
        if (!mbar_wait(&tempty[acc], ((t >> 1) & 1) ^ 1, epi.err, 0x43)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kt = kt0; kt < kt1; ++kt) {
          // One wait: the converter group arrives on a_full only after it has waited for
          // full (the INT8 tile and the token tile landed), so a completed a_full phase
          // orders this step's token tile before the MMAs that read it. (The trace of a
          // step: this thread issuing its MMAs is the step's slowest part.)
          if (!mbar_wait(&a_full[rs], rphase, epi.err, 0x45)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + C::A_COL0 + rs * C::A_COLS;
          const uint32_t b0 = smem_u32(sB + rs * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < kW8K / 16; ++k)  // K = 16 per MMA: 8 TMEM columns of bf16 pairs
            umma_bf16_tmem_a(d_tmem, a_tmem + k * 8,
                             umma_desc_sw128(b0 + (k >> 2) * C::B_HALF + (k & 3) * 32, 16, 1024), idesc,
                             (kt > kt0 || k > 0) ? 1u : 0u);
          umma_commit(&mma_done[rs]);
          if (++rs == RS) {
            rs = 0;
            rphase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, epi.err, 0x46);
    }
  } else if (warp >= 6) {
    // ---------------- INT8 -> bf16 converters. A warp may only reach the TMEM lanes
    // 32 * (warp % 4) ..+31, so lane l of a group's warp w handles weight row
    // 32 * (w % 4) + l of the group's K blocks: kW8K codes read from shared memory,
    // widened, stored as kW8K/2 columns of bf16 pairs.
    const int quarter = warp & 3, group = (warp - 6) >> 2;
    const int r = quarter * 32 + lane;
    // The tile is stored [4 K quarters][128 rows][32 bytes]; a 16-byte access is served
    // per 8 threads (rows r0..r0+7), on 16-byte bank group 2r + chunk (mod 8): rows with
    // bit 2 set read the second chunk of a quarter first, so each phase hits 8 distinct
    // groups.
    const int sw = (r >> 2) & 1;
    const uint32_t raw0 = smem_u32(sRaw) + r * 32;
    const uint32_t lane_addr = ((uint32_t)(quarter * 32) << 16) + C::A_COL0;
    long long i = 0;  // position in the CTA's sequence of K blocks
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int mt, nt, sp, kt0, kt1;
      decode(u, mt, nt, sp, kt0, kt1);
      for (int kt = kt0; kt < kt1; ++kt, ++i) {
        if (i % kW8ConvGroups != group) continue;
        const int rs = (int)(i % RS);
        const uint32_t ph = (uint32_t)((i / RS) & 1);
        // the INT8 tile landed, and the slot's previous MMAs no longer read its TMEM
        if (!mbar_wait_warp(&full[rs], ph, epi.err, 0x47) ||
            !mbar_wait_warp(&mma_done[rs], ph ^ 1, epi.err, 0x48)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t src = raw0 + rs * C::RAW_BYTES;
        const uint32_t dst = tmem_base + lane_addr + rs * C::A_COLS;
#pragma unroll
        for (int hh = 0; hh < C::HALVES; ++hh) {  // K 64*hh .. 64*hh+63
          const uint32_t q0 = src + (2 * hh) * 4096, q1 = q0 + 4096;
          const uint4 c00 = lds128(q0 + sw * 16), c01 = lds128(q0 + (sw ^ 1) * 16);
          const uint4 c10 = lds128(q1 + sw * 16), c11 = lds128(q1 + (sw ^ 1) * 16);
          const uint4 k0 = sw ? c01 : c00, k1 = sw ? c00 : c01;
          const uint4 k2 = sw ? c11 : c10, k3 = sw ? c10 : c11;
          uint32_t p[32];
          i8x4_to_bf16x4(k0.x, p[0], p[1]);
          i8x4_to_bf16x4(k0.y, p[2], p[3]);
          i8x4_to_bf16x4(k0.z, p[4], p[5]);
          i8x4_to_bf16x4(k0.w, p[6], p[7]);
          i8x4_to_bf16x4(k1.x, p[8], p[9]);
          i8x4_to_bf16x4(k1.y, p[10], p[11]);
          i8x4_to_bf16x4(k1.z, p[12], p[13]);
          i8x4_to_bf16x4(k1.w, p[14], p[15]);
          i8x4_to_bf16x4(k2.x, p[16], p[17]);
          i8x4_to_bf16x4(k2.y, p[18], p[19]);
          i8x4_to_bf16x4(k2.z, p[20], p[21]);
          i8x4_to_bf16x4(k2.w, p[22], p[23]);
          i8x4_to_bf16x4(k3.x, p[24], p[25]);
          i8x4_to_bf16x4(k3.y, p[26], p[27]);
          i8x4_to_bf16x4(k3.z, p[28], p[29]);
          i8x4_to_bf16x4(k3.w, p[30], p[31]);
          tmem_st32(dst + hh * 32, reinterpret_cast<const float(&)[32]>(p));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_free[rs]);  // every lane's codes are consumed
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[rs]);
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5): row-scaled split-K partials
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    int t = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++t) {
      int mt, nt, sp, kt0, kt1;
      decode(u, mt, nt, sp, kt0, kt1);
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
  CUtensorMap tb;
  if (reinterpret_cast<uintptr_t>(A8) & 15) return cudaErrorInvalidValue;
  if (!make_tmap_2d_bf16(&tb, B, (uint64_t)N, (uint64_t)K, BN)) return cudaErrorInvalidValue;
  const int KT = (K + kW8K - 1) / kW8K;
  n_split = w8_effective_split(K, n_split);
  const int kt_per = (KT + n_split - 1) / n_split;
  const long long units = (long long)((M + 127) / 128) * n_split;
  const int grid = (int)std::min<long long>(units, num_sms);
  auto kern = gemm_w8_kernel<BN>;
  static std::atomic<unsigned long long> attr_done{0};
  if (cudaError_t e = ensure_smem_attr(kern, C::SMEM, attr_done); e != cudaSuccess)
    return e;
  return launch_k(kern, grid, kW8Threads, C::SMEM, s, (const uint8_t*)A8, tb, row_scale, M, N, K,
                  kt_per, n_split, epi);
}

}  // namespace lb
