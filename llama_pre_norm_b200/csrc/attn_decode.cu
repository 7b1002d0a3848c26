// attn_decode.cu — attention of one decode step over the KV cache ("LLM 核心机制交互讲义",
// chapter 04: y_t = softmax(q_t K_{1:t}^T / sqrt(d_h)) V_{1:t}, only the new token's
// q, k, v are computed; LMDrive page §2.3 for the GQA head grouping).
//
// The step is bound by the HBM read of K and V (each sequence reads
// 2 * (L+1) * H_kv * d_h * 2 bytes), so the kernel is shaped for bandwidth:
//   * split-KV: one CTA per (128-key chunk, KV head, sequence); each CTA moves its
//     K and V chunk (2 x 32 KB, contiguous in the [B, H_kv, t_max, d_h] cache) into
//     shared memory with two bulk async copies, so every byte is read once with
//     full-line transactions and several chunks are in flight per SM;
//   * the n_rep query heads of a KV head share the chunk (GQA without a repeat);
//   * per chunk: scores (thread = key, rotated 16-byte reads of its K row so the
//     warp hits distinct banks), chunk max / sum, then P V (thread = head dim);
//   * a combine kernel merges the per-chunk (max, sum, partial output) triples.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

constexpr int kDecChunk = 128;    // keys per CTA
constexpr int kDecThreads = 128;  // == kDecChunk
constexpr int kMaxRep = 8;        // query heads per KV head handled in one CTA

int decode_attn_chunks(int k_stride) { return (k_stride + kDecChunk - 1) / kDecChunk; }

template <int DH>
__global__ void __launch_bounds__(kDecThreads) attn_decode_split_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
    float* __restrict__ part, int H, int Hkv, int k_stride, int n_chunks,
    const int* __restrict__ kv_len, float scale_log2, int* err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  bf16* sK = reinterpret_cast<bf16*>(smem_raw);
  bf16* sV = sK + kDecChunk * DH;
  float* qs = reinterpret_cast<float*>(sV + kDecChunk * DH);  // [n_rep][DH]
  float* ps = qs + kMaxRep * DH;                               // [n_rep][kDecChunk]
  __shared__ float red[kMaxRep][4];
  __shared__ __align__(8) uint64_t bar;

  const int chunk = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int n_rep = H / Hkv;
  const int nkeys = kv_len[b] + 1;  // cached keys plus the one just appended
  const int c0 = chunk * kDecChunk;
  const int nk = min(kDecChunk, nkeys - c0);
  float* out_base = part + (((long long)b * H + hk * n_rep) * n_chunks + chunk) * (DH + 2);
  const long long head_stride = (long long)n_chunks * (DH + 2);

  if (nk <= 0 || nkeys > k_stride) {
    if (nkeys > k_stride && threadIdx.x == 0 && chunk == 0) latch_error(err, kErrCacheBounds);
    // empty chunk: contributes nothing to the combine
    for (int r = 0; r < n_rep; ++r)
      if (threadIdx.x == 0) {
        out_base[r * head_stride + DH] = -INFINITY;
        out_base[r * head_stride + DH + 1] = 0.f;
      }
    return;
  }

  const long long kv_off = (((long long)b * Hkv + hk) * k_stride + c0) * DH;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    const uint32_t bytes = (uint32_t)nk * DH * 2;
    mbar_arrive_expect_tx(&bar, 2 * bytes);
    bulk_load(sK, k + kv_off, bytes, &bar);
    bulk_load(sV, v + kv_off, bytes, &bar);
  }
  // queries of the n_rep heads, pre-scaled so that scores come out in log2 units
  for (int e = threadIdx.x; e < n_rep * DH; e += kDecThreads) {
    const int r = e / DH, d = e % DH;
    qs[e] = __bfloat162float(q[((long long)b * H + hk * n_rep + r) * DH + d]) * scale_log2;
  }
  __syncthreads();
  // the outcome is made block-uniform so every thread takes the same path
  const bool ok = __syncthreads_and(mbar_wait(&bar, 0, err, 0x31));
  if (!ok) {
    if (threadIdx.x == 0) mbar_wait(&bar, 0, err, 0x32);  // copies in flight must land
    return;
  }

  // scores: thread t scores key c0 + t against every query head of the group
  const int t = threadIdx.x;
  float sc[kMaxRep];
#pragma unroll
  for (int r = 0; r < kMaxRep; ++r) sc[r] = 0.f;
  if (t < nk) {
    const bf16* krow = sK + t * DH;
#pragma unroll 4
    for (int cc = 0; cc < DH / 8; ++cc) {
      const int ch = (cc + t) & (DH / 8 - 1);  // rotate: neighbours read different banks
      float kv8[8];
      load8(krow + ch * 8, kv8);
#pragma unroll
      for (int r = 0; r < kMaxRep; ++r) {
        if (r < n_rep) {
          const float* qq = qs + r * DH + ch * 8;
#pragma unroll
          for (int i = 0; i < 8; ++i) sc[r] = fmaf(qq[i], kv8[i], sc[r]);
        }
      }
    }
  }
  const int lane = t & 31, w = t >> 5;
  // chunk max and sum per head
  float mx[kMaxRep];
#pragma unroll
  for (int r = 0; r < kMaxRep; ++r) {
    float vv = (t < nk && r < n_rep) ? sc[r] : -INFINITY;
    vv = warp_max(vv);
    if (lane == 0) red[r][w] = vv;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kMaxRep; ++r)
    mx[r] = fmaxf(fmaxf(red[r][0], red[r][1]), fmaxf(red[r][2], red[r][3]));
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kMaxRep; ++r) {
    if (r < n_rep) {
      const float p = (t < nk) ? ex2_approx(sc[r] - mx[r]) : 0.f;
      ps[r * kDecChunk + t] = p;
      const float s = warp_sum(p);
      if (lane == 0) red[r][w] = s;
    }
  }
  __syncthreads();
  // P V: thread d accumulates output dimension d (consecutive threads read
  // consecutive bf16 of a V row: conflict-free)
  if (t < DH) {
    for (int r = 0; r < n_rep; ++r) {
      const float* pr = ps + r * kDecChunk;
      float acc = 0.f;
#pragma unroll 8
      for (int j = 0; j < nk; ++j) acc = fmaf(pr[j], __bfloat162float(sV[j * DH + t]), acc);
      float* dst = out_base + r * head_stride;
      dst[t] = acc;
      if (t == 0) {
        dst[DH] = mx[r];
        dst[DH + 1] = red[r][0] + red[r][1] + red[r][2] + red[r][3];
      }
    }
  }
}

// Merge the chunks of one (b, h): M = max_c m_c, l = sum_c l_c 2^(m_c - M),
// o = sum_c o_c 2^(m_c - M) / l.
template <int DH>
__global__ void attn_decode_combine_kernel(const float* __restrict__ part, bf16* __restrict__ o,
                                           int H, int n_chunks, const int* __restrict__ kv_len) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int used = min(n_chunks, (kv_len[b] + 1 + kDecChunk - 1) / kDecChunk);
  const float* base = part + ((long long)b * H + h) * n_chunks * (DH + 2);
  float M = -INFINITY;
  for (int c = 0; c < used; ++c) M = fmaxf(M, base[c * (DH + 2) + DH]);
  float l = 0.f, acc = 0.f;
  for (int c = 0; c < used; ++c) {
    const float* pc = base + c * (DH + 2);
    const float wgt = ex2_approx(pc[DH] - M);
    l += pc[DH + 1] * wgt;
    acc += pc[d] * wgt;
  }
  o[((long long)b * H + h) * DH + d] = __float2bfloat16_rn(acc / l);
}

template <int DH>
static cudaError_t run_decode(const void* q, const void* k, const void* v, void* o, float* part,
                              int B, int H, int Hkv, int k_stride, const int* kv_len, int* err,
                              cudaStream_t s) {
  const int n_chunks = decode_attn_chunks(k_stride);
  const size_t smem = 2 * kDecChunk * DH * 2 + kMaxRep * DH * 4 + kMaxRep * kDecChunk * 4;
  auto kern = attn_decode_split_kernel<DH>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  kern<<<dim3(n_chunks, Hkv, B), kDecThreads, smem, s>>>((const bf16*)q, (const bf16*)k,
                                                         (const bf16*)v, part, H, Hkv, k_stride,
                                                         n_chunks, kv_len, scale_log2, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_decode_combine_kernel<DH><<<dim3(H, B), DH, 0, s>>>(part, (bf16*)o, H, n_chunks, kv_len);
  return cudaGetLastError();
}

cudaError_t launch_attn_decode(const void* q, const void* k, const void* v, void* o, float* part,
                               int B, int H, int Hkv, int dh, int k_stride, const int* kv_len,
                               int* err, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  if (H / Hkv > kMaxRep) return cudaErrorInvalidValue;
  if (dh == 128) return run_decode<128>(q, k, v, o, part, B, H, Hkv, k_stride, kv_len, err, s);
  if (dh == 64) return run_decode<64>(q, k, v, o, part, B, H, Hkv, k_stride, kv_len, err, s);
  return cudaErrorInvalidValue;
}

}  // namespace lb
