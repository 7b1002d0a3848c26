// simt_f32.cu — the fp32 path of the block: plain fp32 FMA kernels (no TF32
// tensor cores, so that the fp32 block keeps fp32 accuracy end to end).
//   * GEMM: nn.Linear y = x W^T (+ residual), LMDrive page §2.3/§2.4.
//   * Causal attention with GQA and an optional per-sequence KV length
//     (prefill and KV-cache decode), LMDrive page §2.3 / mechanics page §02.1 and
//     chapter 04.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

// ---------------------------------------------------------------- GEMM
// 64x64 output tile per 256-thread block, 16-deep K slices staged in shared
// memory (transposed so the inner loop reads broadcast-friendly rows), 4x4
// outputs per thread.
constexpr int kTM = 64, kTN = 64, kTK = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A,
                                                       const float* __restrict__ B,
                                                       float* __restrict__ C,
                                                       const float* __restrict__ resid, int M,
                                                       int N, int K) {
  __shared__ float As[kTK][kTM + 4];
  __shared__ float Bs[kTK][kTN + 4];
  pdl_wait();
  pdl_trigger();
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * kTM, n0 = blockIdx.x * kTN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kTK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = threadIdx.x + r * 256;  // 0..1023 over a 64x16 slice
      const int row = e / kTK, kk = e % kTK;
      const int gm = m0 + row, gn = n0 + row, gk = k0 + kk;
      As[kk][row] = (gm < M && gk < K) ? A[(long long)gm * K + gk] : 0.f;
      Bs[kk][row] = (gn < N && gk < K) ? B[(long long)gn * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kTK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= N) continue;
      const long long o = (long long)gm * N + gn;
      C[o] = resid ? resid[o] + acc[i][j] : acc[i][j];
    }
  }
}

cudaError_t launch_gemm_f32(const float* A, const float* B, float* C, const float* resid, int M,
                            int N, int K, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + kTN - 1) / kTN, (M + kTM - 1) / kTM);
  return launch_k(gemm_f32_kernel, grid, 256, 0, s, A, B, C, resid, M, N, K);
}

// ---------------------------------------------------------------- attention
// One 128-thread block per (query row, head, batch). Keys are visited in chunks
// of 128 with an online softmax: per chunk each thread scores one key, the block
// takes the chunk max, rescales the running sum and output, and each thread
// d < dh accumulates sum_j p_j v_j[d].
constexpr int kAttnThreads = 128;

__global__ void __launch_bounds__(kAttnThreads) attn_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    float* __restrict__ o, int Tq, int Tk, int H, int Hkv, int dh, int k_stride,
    const int* __restrict__ kv_len) {
  __shared__ float qs[128];
  __shared__ float ps[kAttnThreads];
  __shared__ float red[32];
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (H / Hkv);
  const int tk = kv_len ? kv_len[b] + 1 : Tk;
  const int qpos = tk - Tq + i;  // keys 0..qpos are visible
  const float* qrow = q + (((long long)b * H + h) * Tq + i) * dh;
  const float* kb = k + ((long long)b * Hkv + hk) * k_stride * dh;
  const float* vb = v + ((long long)b * Hkv + hk) * k_stride * dh;
  for (int d = threadIdx.x; d < dh; d += kAttnThreads) qs[d] = qrow[d];
  __syncthreads();
  const float scale = 1.0f / sqrtf((float)dh);
  float m_run = -INFINITY, l_run = 0.f, acc = 0.f;  // acc: output dim threadIdx.x
  for (int j0 = 0; j0 <= qpos; j0 += kAttnThreads) {
    const int j = j0 + threadIdx.x;
    float sc = -INFINITY;
    if (j <= qpos) {
      const float* kr = kb + (long long)j * dh;
      float dot = 0.f;
      for (int d = 0; d < dh; ++d) dot = fmaf(qs[d], kr[d], dot);
      sc = dot * scale;
    }
    const float m_new = fmaxf(m_run, block_max(sc, red));
    const float p = (j <= qpos) ? expf(sc - m_new) : 0.f;
    const float alpha = expf(m_run - m_new);  // 0 on the first chunk
    l_run = l_run * alpha + block_sum(p, red);
    ps[threadIdx.x] = p;
    __syncthreads();
    if (threadIdx.x < dh) {
      float s = 0.f;
      const int nj = min(kAttnThreads, qpos + 1 - j0);
      for (int t = 0; t < nj; ++t) s = fmaf(ps[t], vb[(long long)(j0 + t) * dh + threadIdx.x], s);
      acc = acc * alpha + s;
    }
    m_run = m_new;
    __syncthreads();
  }
  if (threadIdx.x < dh) o[(((long long)b * Tq + i) * H + h) * dh + threadIdx.x] = acc / l_run;
}

cudaError_t launch_attn_f32(const float* q, const float* k, const float* v, float* o, int B,
                            int Tq, int Tk, int H, int Hkv, int dh, int k_stride,
                            const int* kv_len, cudaStream_t s) {
  if (B <= 0 || Tq <= 0) return cudaSuccess;
  dim3 grid(Tq, H, B);
  return launch_k(attn_f32_kernel, grid, kAttnThreads, 0, s, q, k, v, o, Tq, Tk, H, Hkv, dh,
                  k_stride, kv_len);
}

}  // namespace lb
