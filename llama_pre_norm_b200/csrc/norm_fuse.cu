// norm_fuse.cu — memory-bound kernels of the block:
//   * RMSNorm (LMDrive page §2.1; "LLM 核心机制交互讲义" §02.3), optionally fused
//     with the residual add of a split-K GEMM's fp32 partial sums,
//   * the QKV finish step (sum of split-K partials, RoPE on Q and K at each
//     token's position, scatter of K/V into the cache) used by decode and by the
//     fp32 path,
//   * SiLU(gate) * up from split-K partials (LlamaMLP, §2.4),
//   * the final residual add (+ cache length increment for decode),
//   * standalone RoPE (rotate_half pairing, §2.2), and rows of the RoPE table for a
//     given rotary base (dynamic NTK scaling).
//
// Every kernel reads 8-element vectors (one 16-byte access for bf16) and
// accumulates in fp32; each stored value is rounded once.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

// ---------------------------------------------------------------- RMSNorm
// One CTA per row. x_row = resid[row] + sum_s partial[s][row] (fp32), rounded to
// T; if x_out: stored there (the residual stream X'). y = g * x_row * r,
// r = 1/sqrt(mean(x_row^2) + eps), computed in fp32, rounded once (g == NULL:
// the gain has been folded into the next GEMM's weights, y = x_row * r).
// Each thread keeps up to kMaxVec 8-element vectors of the row in registers.
constexpr int kNormThreads = 256;
constexpr int kMaxVec = 4;  // rows up to 256 * 8 * 4 = 8192 elements

template <typename T>
__global__ void __launch_bounds__(kNormThreads) resid_rmsnorm_kernel(
    const T* __restrict__ x, const float* __restrict__ partial, int n_split, long long split_stride,
    T* __restrict__ x_out, const T* __restrict__ g, T* __restrict__ y, int d, float eps) {
  __shared__ float red[32];
  pdl_wait();
  pdl_trigger();
  const long long row = blockIdx.x;
  const int nvec = d >> 3;
  float v[kMaxVec][8];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxVec; ++i) {
    const int vi = threadIdx.x + i * kNormThreads;
    if (vi < nvec) {
      load8(x + row * d + vi * 8, v[i]);
      for (int s = 0; s < n_split; ++s) {
        float p[8];
        load8(partial + s * split_stride + row * d + vi * 8, p);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[i][e] += p[e];
      }
      if (n_split > 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[i][e] = round_to<T>(v[i][e]);
        if (x_out) store8(x_out + row * d + vi * 8, v[i]);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += v[i][e] * v[i][e];
    }
  }
  const float r = rsqrtf(block_sum(ss, red) / (float)d + eps);
#pragma unroll
  for (int i = 0; i < kMaxVec; ++i) {
    const int vi = threadIdx.x + i * kNormThreads;
    if (vi < nvec) {
      float gg[8], o[8];
      if (g) {
        load8(g + vi * 8, gg);
      } else {  // gain folded into the consumer's weights
#pragma unroll
        for (int e = 0; e < 8; ++e) gg[e] = 1.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = gg[e] * (v[i][e] * r);
      store8(y + row * d + vi * 8, o);
    }
  }
}

cudaError_t launch_resid_rmsnorm(int dtype, const void* x, const float* partial, int n_split,
                                 long long split_stride, void* x_out, const void* g, void* y,
                                 int rows, int d, float eps, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (dtype == kF32)
    return launch_k(resid_rmsnorm_kernel<float>, rows, kNormThreads, 0, s, (const float*)x, partial,
                    n_split, split_stride, (float*)x_out, (const float*)g, (float*)y, d, eps);
  return launch_k(resid_rmsnorm_kernel<bf16>, rows, kNormThreads, 0, s, (const bf16*)x, partial,
                  n_split, split_stride, (bf16*)x_out, (const bf16*)g, (bf16*)y, d, eps);
}

// ---------------------------------------------------------------- QKV finish
// qkv[s][m][n], n in [0, (H + 2 Hkv) * dh): columns of Q heads, then K, then V
// (the fused projection). Sums the splits, rotates Q and K at position
// pos = pos_base[b] + pos0 + t (row m = b * T + t; pos_base NULL -> 0) using the
// fp32 cos/sin table [max_pos][dh/2], and writes
//   Q -> q_out[b][h][t][:]          ([B, H, T, dh])
//   K -> k_cache[b][hk][pos][:]      ([B, Hkv, t_max, dh]), V likewise.
// One thread per (row, head, pair index i < dh/2).
template <typename T>
__global__ void qkv_finish_kernel(const float* __restrict__ qkv, int n_split,
                                  long long split_stride, int M, int T_, int H, int Hkv, int dh,
                                  const int* __restrict__ pos_base, int pos0,
                                  const float* __restrict__ cos_t,
                                  const float* __restrict__ sin_t, int max_pos, T* __restrict__ q_out,
                                  T* __restrict__ k_cache, T* __restrict__ v_cache, int t_max,
                                  int* err) {
  pdl_wait();
  pdl_trigger();
  const int half = dh >> 1;
  const int heads = H + 2 * Hkv;
  const long long total = (long long)M * heads * half;
  const long long N = (long long)heads * dh;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = idx % half;
    const int hh = (idx / half) % heads;
    const int m = idx / ((long long)half * heads);
    const int b = m / T_, t = m % T_;
    const int pos = (pos_base ? pos_base[b] : 0) + pos0 + t;
    const long long c1 = (long long)hh * dh + i;
    float x1 = 0.f, x2 = 0.f;
    for (int s = 0; s < n_split; ++s) {
      x1 += qkv[s * split_stride + m * N + c1];
      x2 += qkv[s * split_stride + m * N + c1 + half];
    }
    if (hh < H + Hkv) {  // Q or K: rotate
      if (pos < 0 || pos >= max_pos) {
        latch_error(err, kErrPosBounds);
        continue;
      }
      const float c = cos_t[(long long)pos * half + i], sn = sin_t[(long long)pos * half + i];
      const float o1 = x1 * c - x2 * sn, o2 = x2 * c + x1 * sn;
      x1 = o1;
      x2 = o2;
    }
    T* dst;
    if (hh < H) {
      dst = q_out + (((long long)b * H + hh) * T_ + t) * dh;
    } else {
      if (pos < 0 || pos >= t_max) {
        latch_error(err, kErrCacheBounds);
        continue;
      }
      const int hk = hh < H + Hkv ? hh - H : hh - H - Hkv;
      T* base = hh < H + Hkv ? k_cache : v_cache;
      dst = base + (((long long)b * Hkv + hk) * t_max + pos) * dh;
    }
    dst[i] = from_f<T>(x1);
    dst[i + half] = from_f<T>(x2);
  }
}

cudaError_t launch_qkv_finish(int dtype, const float* qkv, int n_split, long long split_stride,
                              int M, int T, int H, int Hkv, int dh, const int* pos_base, int pos0,
                              const float* cos_t, const float* sin_t, int max_pos, void* q_out,
                              void* k_cache, void* v_cache, int t_max, int* err, cudaStream_t s) {
  const long long total = (long long)M * (H + 2 * Hkv) * (dh / 2);
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = (int)std::min<long long>((total + threads - 1) / threads, 148LL * 16);
  if (dtype == kF32)
    return launch_k(qkv_finish_kernel<float>, blocks, threads, 0, s, qkv, n_split, split_stride, M,
                    T, H, Hkv, dh, pos_base, pos0, cos_t, sin_t, max_pos, (float*)q_out,
                    (float*)k_cache, (float*)v_cache, t_max, err);
  return launch_k(qkv_finish_kernel<bf16>, blocks, threads, 0, s, qkv, n_split, split_stride, M, T,
                  H, Hkv, dh, pos_base, pos0, cos_t, sin_t, max_pos, (bf16*)q_out, (bf16*)k_cache,
                  (bf16*)v_cache, t_max, err);
}

// ---------------------------------------------------------------- SiLU * up
// gu[s][m][n'] holds gate and up projections in a packed column order: with
// block == 0 the first f columns are gate and the next f are up; with block > 0
// the columns come in groups of 2*block: [gate block j | up block j]. Writes
// a[m][c] = SiLU(gate) * up, c < f.
template <typename T>
__global__ void silu_mul_kernel(const float* __restrict__ gu, int n_split, long long split_stride,
                                int M, int f, int n_packed, int block, T* __restrict__ a) {
  pdl_wait();
  pdl_trigger();
  const long long total = (long long)M * f;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int c = idx % f;
    const long long m = idx / f;
    long long cg, cu;
    if (block == 0) {
      cg = c;
      cu = (long long)f + c;
    } else {
      cg = (long long)(c / block) * 2 * block + (c % block);
      cu = cg + block;
    }
    float g = 0.f, u = 0.f;
    for (int s = 0; s < n_split; ++s) {
      g += gu[s * split_stride + m * n_packed + cg];
      u += gu[s * split_stride + m * n_packed + cu];
    }
    a[idx] = from_f<T>(silu_f(g) * u);
  }
}

cudaError_t launch_silu_mul(int dtype, const float* gu, int n_split, long long split_stride, int M,
                            int f, int n_packed, int block, void* a, cudaStream_t s) {
  const long long total = (long long)M * f;
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = (int)std::min<long long>((total + threads - 1) / threads, 148LL * 16);
  if (dtype == kF32)
    return launch_k(silu_mul_kernel<float>, blocks, threads, 0, s, gu, n_split, split_stride, M, f,
                    n_packed, block, (float*)a);
  return launch_k(silu_mul_kernel<bf16>, blocks, threads, 0, s, gu, n_split, split_stride, M, f,
                  n_packed, block, (bf16*)a);
}

// ---------------------------------------------------------------- residual add
// out[m][n] = resid[m][n] + sum_s part[s][m][n] (fp32, one rounding). When
// lens != NULL, thread 0..B-1 of block 0 also adds `len_inc` to lens[b].
template <typename T>
__global__ void resid_add_kernel(const T* __restrict__ resid, const float* __restrict__ part,
                                 int n_split, long long split_stride, T* __restrict__ out,
                                 long long total, int* lens, int B, int len_inc) {
  pdl_wait();
  pdl_trigger();
  if (lens && blockIdx.x == 0)
    for (int b = threadIdx.x; b < B; b += blockDim.x) lens[b] += len_inc;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    float v = resid ? to_f<T>(resid[idx]) : 0.f;  // no residual: the partials' sum alone
    for (int s = 0; s < n_split; ++s) v += part[s * split_stride + idx];
    out[idx] = from_f<T>(v);
  }
}

cudaError_t launch_resid_add(int dtype, const void* resid, const float* part, int n_split,
                             long long split_stride, void* out, long long total, int* lens, int B,
                             int len_inc, cudaStream_t s) {
  const int threads = 256;
  const int blocks =
      (int)std::max<long long>(1, std::min<long long>((total + threads - 1) / threads, 148LL * 16));
  if (dtype == kF32)
    return launch_k(resid_add_kernel<float>, blocks, threads, 0, s, (const float*)resid, part,
                    n_split, split_stride, (float*)out, total, lens, B, len_inc);
  return launch_k(resid_add_kernel<bf16>, blocks, threads, 0, s, (const bf16*)resid, part, n_split,
                  split_stride, (bf16*)out, total, lens, B, len_inc);
}

// ---------------------------------------------------------------- row add
// out = a + b row by row (fp32 add, one rounding), and when ss_out != NULL the sum of
// squares of each stored (rounded) out row, the statistic the next GEMM's fused RMSNorm
// reads. Tensor parallelism (Llama-MLP page §6.3): the residual stream plus the
// all-reduced partial sum of a branch.
template <typename T>
__global__ void __launch_bounds__(kNormThreads) add_rows_kernel(const T* __restrict__ a,
                                                                const T* __restrict__ b,
                                                                T* __restrict__ out,
                                                                float* __restrict__ ss_out, int d) {
  __shared__ float red[32];
  pdl_wait();
  pdl_trigger();
  const long long row = blockIdx.x;
  float ss = 0.f;
  for (int vi = threadIdx.x; vi < (d >> 3); vi += kNormThreads) {
    float va[8], vb[8];
    load8(a + row * d + vi * 8, va);
    load8(b + row * d + vi * 8, vb);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      va[e] = round_to<T>(va[e] + vb[e]);
      ss = fmaf(va[e], va[e], ss);
    }
    store8(out + row * d + vi * 8, va);
  }
  if (ss_out) {
    ss = block_sum(ss, red);
    if (threadIdx.x == 0) ss_out[row] = ss;
  }
}

cudaError_t launch_add_rows(int dtype, const void* a, const void* b, void* out, float* ss_out,
                            int rows, int d, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (dtype == kF32)
    return launch_k(add_rows_kernel<float>, rows, kNormThreads, 0, s, (const float*)a,
                    (const float*)b, (float*)out, ss_out, d);
  return launch_k(add_rows_kernel<bf16>, rows, kNormThreads, 0, s, (const bf16*)a, (const bf16*)b,
                  (bf16*)out, ss_out, d);
}

// ---------------------------------------------------------------- row statistics
// Sum of squares of each bf16 row (the RMSNorm statistic; the GEMM that consumes
// the row applies rsqrt(ss/d + eps) in its epilogue). A block takes kSsqRows rows:
// one thread requests them whole from global memory with bulk asynchronous copies
// into shared memory (one mbarrier, bytes counted on completion), then warp w sums
// row w. The copy engine keeps far more bytes in flight per SM than per-thread
// loads can, which is what a read-once kernel needs to reach HBM bandwidth. The kernel
// is bound by the latency of each block's copy, not by DRAM throughput, so the rows go
// one per block (one warp): at the 7B shape 2,048 blocks, all resident at once (10.1
// us against 12.1 with four rows per block and 10.6 with two, same box).
constexpr int kSsqRows = 1;
constexpr int kSsqMaxD = 16384;  // widest row: 32 KB of shared memory per row

__global__ void __launch_bounds__(kSsqRows * 32) row_ssq_kernel(const bf16* __restrict__ x,
                                                                float* __restrict__ ss,
                                                                float* __restrict__ ss_zero,
                                                                int rows, int d, int* lens, int B,
                                                                int len_value, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* buf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const uint32_t row_bytes = (uint32_t)d * 2;
  uint64_t* bar = reinterpret_cast<uint64_t*>(buf + kSsqRows * row_bytes);
  const long long row0 = (long long)blockIdx.x * kSsqRows;
  const int nrows = rows - row0 < kSsqRows ? (int)(rows - row0) : kSsqRows;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  if (lens && blockIdx.x == 0)
    for (int b = threadIdx.x; b < B; b += blockDim.x) lens[b] = len_value;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, (uint32_t)nrows * row_bytes);
    for (int r = 0; r < nrows; ++r)
      bulk_load(buf + r * row_bytes, x + (row0 + r) * d, row_bytes, bar);
  }
  const bool ok = mbar_wait(bar, 0, err, 0x31);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (!ok || w >= nrows) return;
  const uint4* src = reinterpret_cast<const uint4*>(buf + w * row_bytes);
  float acc = 0.f;
  for (int i = lane; i < (d >> 3); i += 32) {
    float v[8];
    unpack_bf16x8(src[i], v);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc = fmaf(v[e], v[e], acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) {
    ss[row0 + w] = acc;
    if (ss_zero) ss_zero[row0 + w] = 0.f;
  }
}

cudaError_t launch_row_ssq(const void* x, float* ss, float* ss_zero, int rows, int d, int* lens,
                           int B, int len_value, int* err, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (d % 8 != 0 || d > kSsqMaxD || (reinterpret_cast<uintptr_t>(x) & 15) != 0)
    return cudaErrorInvalidValue;
  const int smem = kSsqRows * d * 2 + 16 + 128;
  // the limit is raised once per device, so to what the widest supported row needs
  static std::atomic<unsigned long long> attr_done{0};
  if (cudaError_t e = ensure_smem_attr(row_ssq_kernel, kSsqRows * kSsqMaxD * 2 + 16 + 128, attr_done);
      e != cudaSuccess)
    return e;
  return launch_k(row_ssq_kernel, (rows + kSsqRows - 1) / kSsqRows, kSsqRows * 32, smem, s,
                  (const bf16*)x, ss, ss_zero, rows, d, lens, B, len_value, err);
}

// Fold an RMSNorm gain into the weights that consume the normalised row:
// (g * x * r) W^T = r * x (W diag(g))^T.
__global__ void scale_cols_kernel(bf16* __restrict__ w, const bf16* __restrict__ g, long long rows,
                                  int cols) {
  pdl_wait();
  const long long total = rows * cols;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x)
    w[i] = __float2bfloat16_rn(__bfloat162float(w[i]) * __bfloat162float(g[i % cols]));
}

cudaError_t launch_scale_cols(void* w, const void* g, long long rows, int cols, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  return launch_k(scale_cols_kernel, 148 * 16, 256, 0, s, (bf16*)w, (const bf16*)g, rows, cols);
}

// ---------------------------------------------------------------- lengths
__global__ void set_lens_kernel(int* lens, int B, int value) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) lens[b] = value;
}

cudaError_t launch_set_lens(int* lens, int B, int value, cudaStream_t s) {
  return launch_k(set_lens_kernel, (B + 127) / 128, 128, 0, s, lens, B, value);
}

// ---------------------------------------------------------------- RoPE table rows
// Rows [p0, p1) of the RoPE table for rotary base `base` (LMDrive page §2.2
// LlamaRotaryEmbedding: inv_freq_i = base^(-2i/dh), angle = pos * inv_freq_i): the angle
// and its cosine and sine in fp64, stored as fp32 cos / sin [pos][dh/2], the same
// construction as the table the handle builds at creation. Used by dynamic NTK scaling,
// whose base depends on the length a call reaches.
__global__ void rope_table_kernel(float* __restrict__ cos_t, float* __restrict__ sin_t, int p0,
                                  int p1, int half, double base, int dh) {
  pdl_wait();
  pdl_trigger();
  const long long n = (long long)(p1 - p0) * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int p = p0 + (int)(idx / half), i = (int)(idx % half);
    const double inv = 1.0 / pow(base, (2.0 * i) / (double)dh);
    double sv, cv;
    sincos((double)p * inv, &sv, &cv);
    cos_t[(long long)p * half + i] = (float)cv;
    sin_t[(long long)p * half + i] = (float)sv;
  }
}

cudaError_t launch_rope_table(float* cos_t, float* sin_t, int p0, int p1, int half, double base,
                              int dh, cudaStream_t s) {
  if (p1 <= p0 || half <= 0) return cudaSuccess;
  const long long n = (long long)(p1 - p0) * half;
  const int blocks = (int)std::min<long long>((n + 255) / 256, 148 * 8);
  return launch_k(rope_table_kernel, blocks, 256, 0, s, cos_t, sin_t, p0, p1, half, base, dh);
}

// ---------------------------------------------------------------- RoPE (standalone)
// x [B, H, T, dh] rotated in place at positions pos[b][t]. The angle
// pos * base^(-2i/dh) and its sine/cosine are formed in fp64.
template <typename T>
__global__ void rope_apply_kernel(T* __restrict__ x, const int* __restrict__ pos, int B, int T_,
                                  int H, int dh, double base) {
  pdl_wait();
  const int half = dh >> 1;
  const long long total = (long long)B * H * T_ * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = idx % half;
    const long long row = idx / half;  // (b, h, t)
    const int t = row % T_;
    const int b = row / ((long long)T_ * H);
    const double inv = pow(base, -2.0 * (double)i / (double)dh);
    double sd, cd;
    sincos((double)pos[(long long)b * T_ + t] * inv, &sd, &cd);
    const float c = (float)cd, sn = (float)sd;
    T* p = x + row * dh;
    const float x1 = to_f<T>(p[i]), x2 = to_f<T>(p[i + half]);
    p[i] = from_f<T>(x1 * c - x2 * sn);
    p[i + half] = from_f<T>(x2 * c + x1 * sn);
  }
}

cudaError_t launch_rope_apply(int dtype, void* x, const int* pos, int B, int T, int H, int dh,
                              double base, cudaStream_t s) {
  const long long total = (long long)B * H * T * (dh / 2);
  if (total <= 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = (int)std::min<long long>((total + threads - 1) / threads, 148LL * 32);
  if (dtype == kF32)
    rope_apply_kernel<float><<<blocks, threads, 0, s>>>((float*)x, pos, B, T, H, dh, base);
  else
    rope_apply_kernel<bf16><<<blocks, threads, 0, s>>>((bf16*)x, pos, B, T, H, dh, base);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- bounded-wait self-test
// Waits on a barrier that nothing completes; gives up after budget_ns and latches
// the error word. Exercises the same bounded wait every pipelined kernel uses.
__global__ void selftest_timeout_kernel(int* err, unsigned long long budget_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, 0x7f, budget_ns);
  __syncthreads();
}

cudaError_t launch_selftest_timeout(int* err, unsigned long long budget_ns, cudaStream_t s) {
  selftest_timeout_kernel<<<1, 32, 0, s>>>(err, budget_ns);
  return cudaGetLastError();
}

}  // namespace lb
