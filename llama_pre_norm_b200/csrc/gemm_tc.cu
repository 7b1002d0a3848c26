// gemm_tc.cu — bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA, for the four dense contractions of the block (the fused Q|K|V
// projection, o_proj, the fused gate/up projection and down_proj of the
// LlamaAttention / LlamaMLP modules, LMDrive page §2.3–§2.4).
//
//   D[M,N] = A[M,K] · B[N,K]^T        (both operands K-major, fp32 accumulation)
//
// Structure (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: 128x64 A and BNx64 B boxes (128-byte swizzle) into
//               a STAGES-deep shared-memory ring, completion via mbarrier tx counts;
//   warp 1      allocates TMEM, and one thread issues tcgen05.mma (M=128, N=BN,
//               K=16 per instruction) into one of two TMEM accumulators, then
//               tcgen05.commit frees the smem slot / publishes the accumulator;
//   warps 2..5  epilogue: tcgen05.ld (each warp reads its 32-lane TMEM quarter,
//               one output row per thread), fused op, vectorised global stores.
// Two accumulators let the epilogue of tile i overlap the main loop of tile i+1.
//
// Fused epilogues: residual add (o_proj, down_proj: the two residual adds of the
// pre-norm layer, §2.5), SiLU(gate)*up (gate/up rows interleaved in blocks of
// 128 so one 256-wide tile holds matching gate and up columns, §2.4), RoPE on Q
// and K with the scatter of Q into [B,H,T,dh] and K/V into the KV cache (§2.2,
// §2.3), and an fp32 split-K partial store for the swap-AB decode GEMMs.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

constexpr int kBM = 128, kBK = 64;
constexpr int kGemmThreads = 192;
// The pair kernel drains each accumulator with two warps per TMEM lane quarter, each
// taking half of the tile's columns: the epilogue of a pair's last tile is not hidden
// behind another tile's MMAs, and with one warp per quarter it took about half as
// long as the tile's MMAs (a residual epilogue at 256 columns, ~12 us).
constexpr int kPairEpiWarps = 8;
constexpr int kPairThreads = 64 + 32 * kPairEpiWarps;

template <int BN>
struct GemmCfg {
  static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
};

struct Unit {
  int mt, nt, s, kb0, kb1;
};

__device__ __forceinline__ Unit decode_unit(int u, int num_m, int num_n, int KB, int kb_per) {
  Unit r;
  const int mn = num_m * num_n;
  r.s = u / mn;
  const int rem = u - r.s * mn;
  r.mt = rem % num_m;  // m fastest: concurrent CTAs share one weight (B) tile
  r.nt = rem / num_m;
  r.kb0 = r.s * kb_per;
  r.kb1 = min(KB, r.kb0 + kb_per);
  return r;
}

// ------------------------------------------------------------------ epilogues
// RMSNorm statistic of row m folded into the GEMM: rsqrt(mean square + eps), or 1.
__device__ __forceinline__ float row_scale(const GemmEpi& e, int m, int M) {
  if (!e.row_ss || m >= M) return 1.f;
  return rsqrtf(e.row_ss[m] * e.row_inv_d + e.row_eps);
}

// Store 32 consecutive values of one output row at columns [n, n+32) of a row
// with `ncols` columns: vectorised when the whole run is in range, else only
// the in-range elements (ragged last tile).
__device__ __forceinline__ void store_row32(bf16* row, int n, int ncols, const float (&v)[32]) {
  if (n + 32 <= ncols) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float t[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) t[i] = v[q * 8 + i];
      store8(row + n + q * 8, t);
    }
  } else {
    for (int i = 0; i < 32 && n + i < ncols; ++i) row[n + i] = __float2bfloat16_rn(v[i]);
  }
}

// Coalesced output rows for the pair kernel's epilogue warps. A thread owns one output row,
// so a direct 16-byte store of each thread touches 32 rows (32 cache lines) per
// instruction, and those stores slowed the next tile's MMAs. Instead each warp puts two
// 32-column pieces of its 32 rows (two 64-byte segments per row) as bf16 into its own
// 4 KB of shared memory, 16-byte units XOR-swizzled by row (conflict-free on both sides),
// then writes them out with 8 lanes per row: each instruction covers 4 rows x 128 bytes.
constexpr int kStageBytes = 32 * 128;  // per epilogue warp

__device__ __forceinline__ void stage_seg(uint8_t* sw, int lane, int seg, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
    const int unit = seg * 4 + q;
    *reinterpret_cast<uint4*>(sw + lane * 128 + ((unit ^ (lane & 7)) << 4)) = u;
  }
}

// Write the staged rows: segment 0 of row r to row_ptr(r)[0, 32), segment 1 to
// row_ptr(r)[off1, off1 + 32), where row_ptr / ok are this lane's row (lane r owns row r).
__device__ __forceinline__ void stage_flush(const uint8_t* sw, int lane, const bf16* row_ptr, int off1,
                                            bool ok) {
  __syncwarp();
  const unsigned long long p = reinterpret_cast<unsigned long long>(row_ptr);
  const int u = lane & 7;
  const int col = (u >> 2) * off1 + (u & 3) * 8;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = it * 4 + (lane >> 3);
    const uint4 val = *reinterpret_cast<const uint4*>(sw + r * 128 + ((u ^ (r & 7)) << 4));
    bf16* base = reinterpret_cast<bf16*>(__shfl_sync(0xffffffffu, p, r));
    const int okr = __shfl_sync(0xffffffffu, (int)ok, r);
    if (okr) *reinterpret_cast<uint4*>(base + col) = val;
  }
  __syncwarp();  // the buffer may be refilled
}

template <int BN>
__device__ __forceinline__ void epi_store_resid(uint32_t tb, int m, int nt, int M, int N,
                                                const GemmEpi& e, bool with_resid,
                                                int c0 = 0, int c1 = BN / 32) {
  bf16* out = reinterpret_cast<bf16*>(e.out);
  const bf16* res = reinterpret_cast<const bf16*>(e.resid);
  float ssq = 0.f;
#pragma unroll 1
  for (int c = c0; c < c1; ++c) {
    float v[32];
    tmem_ld32(tb + c * 32, v);
    tmem_wait_ld();
    const int n = nt * BN + c * 32;
    if (m < M && n < N) {
      const long long o = (long long)m * e.ldo;
      if (with_resid) {
        if (n + 32 <= N) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float r[8];
            load8(res + o + n + q * 8, r);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[q * 8 + i] += r[i];
          }
        } else {
          for (int i = 0; i < 32 && n + i < N; ++i) v[i] += __bfloat162float(res[o + n + i]);
        }
      }
      if (e.ss_out) {  // statistic of the stored (rounded) row for the next RMSNorm
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          v[i] = round_to<bf16>(v[i]);
          if (n + i < N) ssq += v[i] * v[i];
        }
      }
      store_row32(out + o, n, N, v);
    }
  }
  if (e.ss_out && m < M) atomicAdd(e.ss_out + m, ssq);
}

// Residual-add epilogue with the row's residual already in registers (rres: the
// BN columns of row m, loaded before the accumulator was ready).
template <int BN, int NC>
__device__ __forceinline__ void prefetch_resid(uint4 (&rres)[NC / 8], int m, int nt, int M, int N,
                                               const GemmEpi& e, int c0) {
  const int n0 = nt * BN;
  if (m < M && n0 + BN <= N) {
    const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const bf16*>(e.resid) +
                                                      (long long)m * e.ldo + n0 + c0 * 32);
#pragma unroll
    for (int i = 0; i < NC / 8; ++i) rres[i] = src[i];
  }
}

template <int BN, int NC>
__device__ __forceinline__ void epi_resid_prefetched(uint32_t tb, int m, int nt, int M, int N,
                                                     const GemmEpi& e, const uint4 (&rres)[NC / 8],
                                                     int c0, uint8_t* stage, int lane) {
  const int n0 = nt * BN;
  // ragged tile (some row of this warp or the columns out of range): the general
  // path. The choice is warp-uniform: tcgen05.ld is a warp-collective instruction.
  if (!__all_sync(0xffffffffu, m < M && n0 + BN <= N)) {
    epi_store_resid<BN>(tb, m, nt, M, N, e, true, c0, c0 + NC / 32);
    return;
  }
  bf16* out = reinterpret_cast<bf16*>(e.out) + (long long)m * e.ldo;
  float ssq = 0.f;
#pragma unroll  // static indices keep rres in registers
  for (int cc = 0; cc < NC / 32; ++cc) {
    const int c = c0 + cc;
    float v[32];
    tmem_ld32(tb + c * 32, v);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float r[8];
      unpack_bf16x8(rres[cc * 4 + q], r);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[q * 8 + i] += r[i];
    }
    if (e.ss_out) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        v[i] = round_to<bf16>(v[i]);
        ssq += v[i] * v[i];
      }
    }
    stage_seg(stage, lane, cc & 1, v);
    if (cc & 1) stage_flush(stage, lane, out + n0 + (c - 1) * 32, 32, true);
  }
  if (e.ss_out && m < M) atomicAdd(e.ss_out + m, ssq);
}

// Tile columns [0,128) are gate rows 128*nt.., [128,256) the matching up rows.
__device__ __forceinline__ void epi_swiglu(uint32_t tb, int m, int nt, int M, int f,
                                           const GemmEpi& e, int j0 = 0, int j1 = 4,
                                           uint8_t* stage = nullptr, int lane = 0) {
  bf16* out = reinterpret_cast<bf16*>(e.out);
  const float r = row_scale(e, m, M);
  // staged, coalesced stores when the warp's columns are whole pairs of chunks in range
  if (stage && ((j1 - j0) & 1) == 0 && nt * 128 + j1 * 32 <= f) {
    bf16* row = out + (long long)m * e.ldo;
#pragma unroll 1
    for (int j = j0; j < j1; ++j) {
      float g[32], u[32];
      tmem_ld32(tb + j * 32, g);
      tmem_ld32(tb + 128 + j * 32, u);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i] * r) * (u[i] * r);
      stage_seg(stage, lane, (j - j0) & 1, g);
      if ((j - j0) & 1) stage_flush(stage, lane, row + nt * 128 + (j - 1) * 32, 32, m < M);
    }
    return;
  }
#pragma unroll 1
  for (int j = j0; j < j1; ++j) {
    float g[32], u[32];
    tmem_ld32(tb + j * 32, g);
    tmem_ld32(tb + 128 + j * 32, u);
    tmem_wait_ld();
    const int col = nt * 128 + j * 32;
    if (m < M && col < f) {
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i] * r) * (u[i] * r);
      store_row32(out + (long long)m * e.ldo, col, f, g);
    }
  }
}

// Columns of the fused projection: Q heads [0, H*dh), K heads, then V heads.
// Each thread owns token row m = b*T + t at position pos0 + t; RoPE pairs column i with
// i + dh/2 of the same head (rotate_half), both held by this thread.
template <int BN>
__device__ __forceinline__ void epi_qkv_rope(uint32_t tb, int m, int nt, int M, int N,
                                             const GemmEpi& e, int part = 0, int nparts = 1,
                                             uint8_t* stage = nullptr, int lane = 0) {
  const int dh = e.dh, half = dh >> 1;
  const int b = m / e.T, t = m - (m / e.T) * e.T;
  const int pos = e.pos0 + t;
  const bool row_ok = m < M;
  const float r = row_scale(e, m, M);
  bool pos_ok = pos < e.max_pos && pos < e.t_max;
  if (row_ok && !pos_ok && part == 0) latch_error(e.err, kErrCacheBounds);
  // heads of the tile taken by this part (BN / dh is 2 or 4, nparts 1 or 2)
  const int nh = BN / dh, h0 = part * nh / nparts, h1 = (part + 1) * nh / nparts;
#pragma unroll 1
  for (int hh = h0; hh < h1; ++hh) {
    const int gcol = nt * BN + hh * dh;
    if (gcol >= N) break;  // uniform across the warp
    const int hq = gcol / dh;
    bf16* dst;
    bool rotate = true;
    if (hq < e.H) {
      dst = reinterpret_cast<bf16*>(e.q_out) + (((long long)b * e.H + hq) * e.T + t) * dh;
    } else if (hq < e.H + e.Hkv) {
      dst = reinterpret_cast<bf16*>(e.k_cache) +
            (((long long)b * e.Hkv + (hq - e.H)) * e.t_max + pos) * dh;
    } else {
      dst = reinterpret_cast<bf16*>(e.v_cache) +
            (((long long)b * e.Hkv + (hq - e.H - e.Hkv)) * e.t_max + pos) * dh;
      rotate = false;
    }
    const bool store = row_ok && pos_ok;
    if (stage) {  // staged, coalesced stores (every thread takes part; `store` masks rows)
      if (rotate) {
#pragma unroll 1
        for (int j = 0; j < half / 32; ++j) {
          float x1[32], x2[32];
          tmem_ld32(tb + hh * dh + j * 32, x1);
          tmem_ld32(tb + hh * dh + half + j * 32, x2);
          tmem_wait_ld();
          const float* ct = e.cos_t + (long long)(store ? pos : 0) * half + j * 32;
          const float* st = e.sin_t + (long long)(store ? pos : 0) * half + j * 32;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float c[8], sn[8];
            load8(ct + q * 8, c);
            load8(st + q * 8, sn);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float a = x1[q * 8 + i] * r, bb = x2[q * 8 + i] * r;
              x1[q * 8 + i] = a * c[i] - bb * sn[i];
              x2[q * 8 + i] = bb * c[i] + a * sn[i];
            }
          }
          stage_seg(stage, lane, 0, x1);
          stage_seg(stage, lane, 1, x2);
          stage_flush(stage, lane, dst + j * 32, half, store);
        }
      } else {
#pragma unroll 1
        for (int j = 0; j < dh / 32; ++j) {
          float x[32];
          tmem_ld32(tb + hh * dh + j * 32, x);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] *= r;
          stage_seg(stage, lane, j & 1, x);
          if (j & 1) stage_flush(stage, lane, dst + (j - 1) * 32, 32, store);
        }
      }
    } else if (rotate) {
#pragma unroll 1
      for (int j = 0; j < half / 32; ++j) {
        float x1[32], x2[32];
        tmem_ld32(tb + hh * dh + j * 32, x1);
        tmem_ld32(tb + hh * dh + half + j * 32, x2);
        tmem_wait_ld();
        if (store) {
          const float* ct = e.cos_t + (long long)pos * half + j * 32;
          const float* st = e.sin_t + (long long)pos * half + j * 32;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float c[8], s[8], o1[8], o2[8];
            load8(ct + q * 8, c);
            load8(st + q * 8, s);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float a = x1[q * 8 + i] * r, bb = x2[q * 8 + i] * r;
              o1[i] = a * c[i] - bb * s[i];
              o2[i] = bb * c[i] + a * s[i];
            }
            store8(dst + j * 32 + q * 8, o1);
            store8(dst + half + j * 32 + q * 8, o2);
          }
        }
      }
    } else {
#pragma unroll 1
      for (int j = 0; j < dh / 32; ++j) {
        float x[32];
        tmem_ld32(tb + hh * dh + j * 32, x);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = x[q * 8 + i] * r;
            store8(dst + j * 32 + q * 8, o);
          }
        }
      }
    }
  }
}

// Swap-AB decode: rows are weight rows (output features), columns are tokens.
// part[s][token][row] = acc, so that a warp's 32 lanes write 32 consecutive floats.
template <int BN>
__device__ __forceinline__ void epi_partial_t(uint32_t tb, int row, int nt, int s, int M, int N,
                                              const GemmEpi& e) {
  float* part = reinterpret_cast<float*>(e.out) + (long long)s * e.split_stride;
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    float v[32];
    tmem_ld32(tb + c * 32, v);
    tmem_wait_ld();
    if (row < M) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int tok = nt * BN + c * 32 + i;
        if (tok < N) part[(long long)tok * e.ldo + row] = v[i];
      }
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int BN, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   int M, int N, int K, int kb_per, int n_split, GemmEpi epi) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Inputs of the previous kernel are complete and visible after pdl_wait. The weight
  // operand (A in the swap-AB decode form, B otherwise) is no such input: the producer
  // fills the ring with the first weight tiles before it waits.
  if (warp != 0) pdl_wait();

  const int num_m = (M + kBM - 1) / kBM, num_n = (N + BN - 1) / BN;
  const int KB = (K + kBK - 1) / kBK;
  const int units = num_m * num_n * n_split;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      constexpr bool kAIsWeight = EPI == kEpiPartialT;
      int npre = 0;  // leading k-blocks of the first unit whose weight tile is in flight
      if ((int)blockIdx.x < units) {
        const Unit w = decode_unit(blockIdx.x, num_m, num_n, KB, kb_per);
        npre = min(w.kb1 - w.kb0, C::STAGES);
        for (int i = 0; i < npre; ++i) {  // fresh ring: stage i is free
          const int kb = w.kb0 + i;
          mbar_arrive_expect_tx(&full[i], C::STAGE_BYTES);
          if (kAIsWeight)
            tma_load_2d(sA + i * C::A_BYTES, &tmA, &full[i], kb * kBK, w.mt * kBM);
          else
            tma_load_2d(sB + i * C::B_BYTES, &tmB, &full[i], kb * kBK, w.nt * BN);
        }
      }
      pdl_wait();
      uint32_t stage = 0, phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Unit w = decode_unit(u, num_m, num_n, KB, kb_per);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          const bool pre = issued < npre;  // weight tile already requested above
          if (!pre) {
            if (!mbar_wait(&empty[stage], phase ^ 1, epi.err, 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          }
          if (!pre || !kAIsWeight)
            tma_load_2d(sA + stage * C::A_BYTES, &tmA, &full[stage], kb * kBK, w.mt * kBM);
          if (!pre || kAIsWeight)
            tma_load_2d(sB + stage * C::B_BYTES, &tmB, &full[stage], kb * kBK, w.nt * BN);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      pdl_trigger();  // all loads issued: the next kernel may start launching
      // Every load issued must land before the CTA may exit.
      const long long first = issued > C::STAGES ? issued - C::STAGES : 0;
      for (long long i = first; i < issued; ++i)
        mbar_wait(&full[i % C::STAGES], (uint32_t)((i / C::STAGES) & 1), epi.err, 6);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc = umma_idesc_bf16(kBM, BN, 0, 0);
      uint32_t stage = 0, phase = 0;
      int t = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++t) {
        const Unit w = decode_unit(u, num_m, num_n, KB, kb_per);
        const int acc = t & 1;
        if (!mbar_wait(&tempty[acc], ((t >> 1) & 1) ^ 1, epi.err, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, epi.err, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t ad = umma_desc_sw128(a0 + k * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(b0 + k * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (kb > w.kb0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      // All issued MMAs must complete before TMEM is released.
      umma_commit(drain);
      mbar_wait(drain, 0, epi.err, 4);
    }
  } else {
    // ---------------- epilogue (warps 2..5)
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row_in_tile = quarter * 32 + lane;
    int t = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++t) {
      const Unit w = decode_unit(u, num_m, num_n, KB, kb_per);
      const int acc = t & 1;
      if (!mbar_wait_warp(&tfull[acc], (t >> 1) & 1, epi.err, 5)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      const int m = w.mt * kBM + row_in_tile;
      if constexpr (EPI == kEpiStore) {
        epi_store_resid<BN>(tb, m, w.nt, M, N, epi, false);
      } else if constexpr (EPI == kEpiResid) {
        epi_store_resid<BN>(tb, m, w.nt, M, N, epi, true);
      } else if constexpr (EPI == kEpiSwiGLU) {
        epi_swiglu(tb, m, w.nt, M, epi.f, epi);
      } else if constexpr (EPI == kEpiQkvRope) {
        epi_qkv_rope<BN>(tb, m, w.nt, M, N, epi);
      } else {
        epi_partial_t<BN>(tb, m, w.nt, w.s, M, N, epi);
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

// ------------------------------------------------------------------ 2-SM pair kernel
// The same GEMM with 256 x BN tiles computed by a cluster of two CTAs: CTA r of the
// pair loads rows [128r, 128r+128) of the A tile and rows [r BN/2, (r+1) BN/2) of
// the B tile into its own shared memory (32 KB per k-block at BN = 256, so six
// stages fit), the even CTA issues tcgen05.mma.cta_group::2 (M = 256) which reads
// both CTAs' operands and leaves each CTA's 128 accumulator rows in its own TMEM,
// and both CTAs run the epilogue on their rows. Per SM the operand traffic per
// MMA is two thirds of the 1-SM 128 x 256 tile's.
template <int BN>
struct Gemm2Cfg {
  static constexpr int STAGES = 6;
  static constexpr int A_BYTES = 128 * kBK * 2;
  static constexpr int B_BYTES = (BN / 2) * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int OUT_STAGE = kPairEpiWarps * kStageBytes;  // coalesced output rows
  static constexpr int SMEM = STAGES * STAGE_BYTES + 256 + OUT_STAGE + 1024;
  static_assert(SMEM <= 232448, "pair GEMM exceeds the shared memory of a CTA");
};

template <int BN, int EPI>
__global__ void __launch_bounds__(kPairThreads, 1)
    gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, int M, int N, int K, GemmEpi epi) {
  using C = Gemm2Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                  // used in the leader: both CTAs' bytes
  uint64_t* empty = bars + C::STAGES;     // each CTA: its stage may be refilled
  uint64_t* tfull = bars + 2 * C::STAGES; // each CTA: accumulator ready
  uint64_t* tempty = tfull + 2;           // leader: both CTAs drained the accumulator
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kPairEpiWarps);  // epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (warp >= 2 || (warp == 1 && !epi.operands_ready)) pdl_wait();

  const int num_m = (M + 2 * kBM - 1) / (2 * kBM), num_n = (N + BN - 1) / BN;
  const int KB = (K + kBK - 1) / kBK;
  const int units = num_m * num_n;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      // The weight operand B is no output of the previous kernel: the B tiles of the
      // first ring's worth of K blocks are requested before waiting for that kernel;
      // their A tiles (the activations) follow once it has completed.
      int npre = 0;
      if (pair < units) {
        const int nt0 = pair / num_m;
        npre = min(KB, C::STAGES);
        for (int kb = 0; kb < npre; ++kb) {  // fresh ring: every stage is free
          if (rank == 0) mbar_arrive_expect_tx(&full[kb], 2 * C::STAGE_BYTES);
          tma_load_2d_pair(sB + kb * C::B_BYTES, &tmB, pair_addr(&full[kb], 0), kb * kBK,
                           nt0 * BN + rank * (BN / 2));
        }
      }
      if (!epi.operands_ready) pdl_wait();
      uint32_t stage = 0, phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int u = pair; u < units && ok; u += npairs) {
        const int mt = u % num_m, nt = u / num_m;
        for (int kb = 0; kb < KB; ++kb) {
          const uint32_t fb = pair_addr(&full[stage], 0);
          if (issued < npre) {  // B already requested
            tma_load_2d_pair(sA + stage * C::A_BYTES, &tmA, fb, kb * kBK, mt * 2 * kBM + rank * kBM);
          } else {
            if (!mbar_wait(&empty[stage], phase ^ 1, epi.err, 0x11)) {
              ok = false;
              break;
            }
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
            tma_load_2d_pair(sA + stage * C::A_BYTES, &tmA, fb, kb * kBK, mt * 2 * kBM + rank * kBM);
            tma_load_2d_pair(sB + stage * C::B_BYTES, &tmB, fb, kb * kBK, nt * BN + rank * (BN / 2));
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      pdl_trigger();
      // The last loads must have landed and been consumed before the pair may exit.
      const long long first = issued > C::STAGES ? issued - C::STAGES : 0;
      for (long long i = first; i < issued; ++i)
        mbar_wait(&empty[i % C::STAGES], (uint32_t)((i / C::STAGES) & 1), epi.err, 0x12);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader CTA)
      constexpr uint32_t idesc = umma_idesc_bf16(2 * kBM, BN, 0, 0);
      uint32_t stage = 0, phase = 0;
      int t = 0;
      bool ok = true;
      for (int u = pair; u < units && ok; u += npairs, ++t) {
        const int acc = t & 1;
        if (!mbar_wait(&tempty[acc], ((t >> 1) & 1) ^ 1, epi.err, 0x13)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, epi.err, 0x14)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16_pair(d_tmem, umma_desc_sw128(a0 + k * 32, 16, 1024),
                           umma_desc_sw128(b0 + k * 32, 16, 1024), idesc, (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit_pair(pair_addr(&empty[stage], 0));
          umma_commit_pair(pair_addr(&empty[stage], 1));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(pair_addr(&tfull[acc], 0));
        umma_commit_pair(pair_addr(&tfull[acc], 1));
      }
      umma_commit_pair(pair_addr(drain, 0));
      mbar_wait(drain, 0, epi.err, 0x15);
    }
  } else {
    // ---------------- epilogue (warps 2.. of both CTAs, 128 rows each): warp w reads
    // TMEM lane quarter w % 4 and takes part (w - 2) / 4 of the tile's columns
    constexpr int kParts = kPairEpiWarps / 4;
    const int quarter = warp & 3, part = (warp - 2) >> 2;
    const int row_in_tile = quarter * 32 + lane;
    constexpr int NC = BN / kParts;  // columns per part
    const int c0 = part * (NC / 32);
    uint8_t* stage = smem + C::STAGES * C::STAGE_BYTES + 256 + (warp - 2) * kStageBytes;
    int t = 0;
    for (int u = pair; u < units; u += npairs, ++t) {
      const int mt = u % num_m, nt = u / num_m;
      const int acc = t & 1;
      const int m = mt * 2 * kBM + rank * kBM + row_in_tile;
      // The residual is fetched while the accumulator is still being computed.
      const bool prefetch = EPI == kEpiResid;
      uint4 rres[EPI == kEpiResid ? NC / 8 : 1];
      if constexpr (EPI == kEpiResid)
        if (prefetch) prefetch_resid<BN, NC>(rres, m, nt, M, N, epi, c0);
      if (!mbar_wait_warp(&tfull[acc], (t >> 1) & 1, epi.err, 0x16)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      if constexpr (EPI == kEpiStore) {
        epi_store_resid<BN>(tb, m, nt, M, N, epi, false, c0, c0 + NC / 32);
      } else if constexpr (EPI == kEpiResid) {
        if (prefetch)
          epi_resid_prefetched<BN, NC>(tb, m, nt, M, N, epi, rres, c0, stage, lane);
        else
          epi_store_resid<BN>(tb, m, nt, M, N, epi, true, c0, c0 + NC / 32);
      } else if constexpr (EPI == kEpiSwiGLU) {
        epi_swiglu(tb, m, nt, M, epi.f, epi, part * 4 / kParts, (part + 1) * 4 / kParts, stage, lane);
      } else {
        epi_qkv_rope<BN>(tb, m, nt, M, N, epi, part, kParts, stage, lane);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(pair_addr(&tempty[acc], 0));
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();  // the leader's MMAs have finished reading both CTAs' operands
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
template <int BN, int EPI>
static cudaError_t run(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                       int kb_per, int n_split, const GemmEpi& epi, int grid, cudaStream_t s) {
  using C = GemmCfg<BN>;
  auto kern = gemm_tc_kernel<BN, EPI>;
  static std::atomic<unsigned long long> attr_done{0};
  if (cudaError_t e = ensure_smem_attr(kern, C::SMEM, attr_done); e != cudaSuccess)
    return e;
  return launch_k(kern, grid, kGemmThreads, C::SMEM, s, ta, tb, M, N, K, kb_per, n_split, epi);
}

template <int BN, int EPI>
static cudaError_t run_pair(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                            const GemmEpi& epi, int grid, cudaStream_t s) {
  using C = Gemm2Cfg<BN>;
  auto kern = gemm_tc_pair_kernel<BN, EPI>;
  static std::atomic<unsigned long long> attr_done{0};
  if (cudaError_t e = ensure_smem_attr(kern, C::SMEM, attr_done); e != cudaSuccess)
    return e;
  return launch_k_pair(kern, grid, kPairThreads, C::SMEM, s, ta, tb, M, N, K, epi);
}

// 2-SM pair path: 256 x 256 tiles, no split-K.
static cudaError_t launch_gemm_tc_pair(const void* A, const void* B, int M, int N, int K,
                                      const GemmEpi& epi, int num_sms, cudaStream_t s) {
  CUtensorMap ta, tb;
  if (!make_tmap_2d_bf16(&ta, A, (uint64_t)M, (uint64_t)K, kBM)) return cudaErrorInvalidValue;
  if (!make_tmap_2d_bf16(&tb, B, (uint64_t)N, (uint64_t)K, 128)) return cudaErrorInvalidValue;
  const long long units = (long long)((M + 255) / 256) * ((N + 255) / 256);
  const int grid = (int)std::min<long long>(2 * units, num_sms & ~1);
  switch (epi.kind) {
    case kEpiStore: return run_pair<256, kEpiStore>(ta, tb, M, N, K, epi, grid, s);
    case kEpiResid: return run_pair<256, kEpiResid>(ta, tb, M, N, K, epi, grid, s);
    case kEpiSwiGLU: return run_pair<256, kEpiSwiGLU>(ta, tb, M, N, K, epi, grid, s);
    case kEpiQkvRope: return run_pair<256, kEpiQkvRope>(ta, tb, M, N, K, epi, grid, s);
  }
  return cudaErrorInvalidConfiguration;
}

cudaError_t launch_gemm_tc(const void* A, const void* B, int M, int N, int K, int BN, int n_split,
                           const GemmEpi& epi, int num_sms, cudaStream_t s) {
  if (M <= 0 || N <= 0 || K <= 0) return cudaSuccess;
  // Prefill-sized GEMMs run on CTA pairs (2-SM MMA, 256 x 256 tiles).
  if (BN == 256 && n_split == 1 && epi.kind != kEpiPartialT && M > 128 && num_sms >= 2)
    return launch_gemm_tc_pair(A, B, M, N, K, epi, num_sms, s);
  CUtensorMap ta, tb;
  if (!make_tmap_2d_bf16(&ta, A, (uint64_t)M, (uint64_t)K, kBM)) return cudaErrorInvalidValue;
  if (!make_tmap_2d_bf16(&tb, B, (uint64_t)N, (uint64_t)K, (uint32_t)BN))
    return cudaErrorInvalidValue;
  const int KB = (K + kBK - 1) / kBK;
  n_split = gemm_effective_split(K, n_split);
  const int kb_per = (KB + n_split - 1) / n_split;
  const long long units =
      (long long)((M + kBM - 1) / kBM) * ((N + BN - 1) / BN) * (long long)n_split;
  const int grid = (int)std::min<long long>(units, num_sms);
  switch (epi.kind) {
    case kEpiStore:
      if (BN == 256) return run<256, kEpiStore>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      if (BN == 128) return run<128, kEpiStore>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      break;
    case kEpiResid:
      if (BN == 256) return run<256, kEpiResid>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      if (BN == 128) return run<128, kEpiResid>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      break;
    case kEpiSwiGLU:
      if (BN == 256) return run<256, kEpiSwiGLU>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      break;
    case kEpiQkvRope:
      if (BN == 256) return run<256, kEpiQkvRope>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      break;
    case kEpiPartialT:
      if (BN == 32) return run<32, kEpiPartialT>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      if (BN == 64) return run<64, kEpiPartialT>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      if (BN == 128) return run<128, kEpiPartialT>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      if (BN == 256) return run<256, kEpiPartialT>(ta, tb, M, N, K, kb_per, n_split, epi, grid, s);
      break;
  }
  return cudaErrorInvalidConfiguration;
}

}  // namespace lb
