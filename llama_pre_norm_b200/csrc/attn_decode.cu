// attn_decode.cu — attention of one decode step over the KV cache ("LLM 核心机制交互讲义",
// chapter 04: y_t = softmax(q_t K_{1:t}^T / sqrt(d_h)) V_{1:t}, only the new token's
// q, k, v are computed; LMDrive page §2.3 for the GQA head grouping).
//
// The step is bound by the HBM read of K and V (each sequence reads
// 2 * (L+1) * H_kv * d_h * 2 bytes), so the kernel is shaped to keep HBM busy:
//   * split-KV: one CTA per (512-key split, group of G query heads, sequence);
//   * a producer warp streams the split through a 3-stage shared-memory ring of
//     64-key chunks (K and V rows are contiguous in the [B, H_kv, t_max, d_h]
//     cache, so each chunk is two bulk async copies), while
//   * eight consumer warps each own 8 keys of every chunk and keep their own
//     online-softmax state (running max, sum and output) for G query heads of the
//     KV head, so no block-wide reduction sits inside the key loop. G is the
//     largest of 8, 4, 2, 1 that divides n_rep = H / H_kv, so one CTA serves the
//     whole group when n_rep is 1, 2, 4 or 8 and n_rep / G CTAs share it otherwise
//     (any n_rep works; for n_rep = 3, 5, ... each CTA serves one query head):
//       scores: lane = (key, quarter of d_h); 16-byte K reads rotated per lane so a
//               quarter-warp hits 8 different banks; q held pre-rotated in registers;
//       P V:    lane = d_h/32 consecutive dims; a warp reads whole V rows;
//   * the warps' states are merged in shared memory and one (max, sum, output)
//     partial per (split, head) goes to global memory; a combine kernel merges the
//     splits of each (sequence, head).
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

constexpr int kDecChunk = 64;         // keys per pipeline stage
constexpr int kDecStages = 3;
constexpr int kDecSplitKeys = 512;    // keys per CTA
constexpr int kDecWarps = 8;          // consumer warps (8 keys of each chunk apiece)
constexpr int kDecThreads = (kDecWarps + 1) * 32;

int decode_attn_chunks(int k_stride) { return (k_stride + kDecSplitKeys - 1) / kDecSplitKeys; }

int decode_attn_heads_per_cta(int n_rep) {
  return n_rep % 8 == 0 ? 8 : n_rep % 4 == 0 ? 4 : n_rep % 2 == 0 ? 2 : 1;
}

template <int DH>
constexpr int dec_smem_bytes(int nrep) {
  return kDecStages * 2 * kDecChunk * DH * 2 + nrep * DH * 4;
}

template <int DH, int NREP>
__global__ void __launch_bounds__(kDecThreads, NREP >= 4 ? 1 : 2) attn_decode_split_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
    float* __restrict__ part, int H, int Hkv, int k_stride, int n_splits,
    const int* __restrict__ kv_len, float scale_log2, int* err) {
  // NREP: query heads of this CTA (G above); they are heads hq0 .. hq0 + NREP - 1,
  // all in the group of KV head hk.
  constexpr int QD = DH / 4;           // dims per lane in the score phase
  constexpr int QC = QD / 8;           // 16-byte chunks per lane (4 or 2)
  constexpr int VD = DH / 32;          // dims per lane in the P V phase (4 or 2)
  constexpr int CHUNK_BYTES = kDecChunk * DH * 2;
  constexpr bool Q_IN_REGS = NREP <= 2;
  extern __shared__ __align__(128) uint8_t smem[];
  bf16* sKV = reinterpret_cast<bf16*>(smem);  // stage s: K at 2s, V at 2s+1 (CHUNK_BYTES each)
  float* qs = reinterpret_cast<float*>(smem + kDecStages * 2 * CHUNK_BYTES);  // [NREP][DH]
  __shared__ __align__(8) uint64_t full[kDecStages], empty[kDecStages];

  pdl_wait();
  pdl_trigger();
  const int split = blockIdx.x, b = blockIdx.z;
  const int hq0 = blockIdx.y * NREP;
  const int hk = hq0 / (H / Hkv);
  const int nkeys = kv_len[b] + 1;  // cached keys plus the one just appended
  const int k0 = split * kDecSplitKeys;
  const int nk = min(kDecSplitKeys, nkeys - k0);
  const long long head_stride = (long long)n_splits * (DH + 2);
  float* out_base = part + (((long long)b * H + hq0) * n_splits + split) * (DH + 2);

  if (nk <= 0 || nkeys > k_stride) {
    // a length outside [0, k_stride) is an error; the split then reads nothing
    if ((nkeys > k_stride || nkeys <= 0) && threadIdx.x == 0 && split == 0)
      latch_error(err, kErrCacheBounds);
    if (threadIdx.x < NREP) {  // empty split: contributes nothing to the combine
      out_base[threadIdx.x * head_stride + DH] = -INFINITY;
      out_base[threadIdx.x * head_stride + DH + 1] = 0.f;
    }
    return;
  }
  const int nch = (nk + kDecChunk - 1) / kDecChunk;
  const long long kv_off = (((long long)b * Hkv + hk) * k_stride + k0) * DH;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecWarps);
    }
    fence_mbar_init();
  }
  for (int e = threadIdx.x; e < NREP * DH; e += kDecThreads)
    qs[e] = __bfloat162float(q[((long long)b * H + hq0) * DH + e]) * scale_log2;
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == kDecWarps) {
    // ---------------- producer: stream the split through the ring
    if (lane == 0) {
      int issued = 0;
      for (int c = 0; c < nch; ++c) {
        const int st = c % kDecStages;
        if (c >= kDecStages && !mbar_wait(&empty[st], ((c / kDecStages) - 1) & 1, err, 0x33)) break;
        const int rows = min(kDecChunk, nk - c * kDecChunk);
        const uint32_t bytes = (uint32_t)rows * DH * 2;
        mbar_arrive_expect_tx(&full[st], 2 * bytes);
        const long long off = kv_off + (long long)c * kDecChunk * DH;
        bulk_load(sKV + (2 * st) * (CHUNK_BYTES / 2), k + off, bytes, &full[st]);
        bulk_load(sKV + (2 * st + 1) * (CHUNK_BYTES / 2), v + off, bytes, &full[st]);
        issued = c + 1;
      }
      for (int c = max(0, issued - kDecStages); c < issued; ++c)  // copies must land before exit
        mbar_wait(&full[c % kDecStages], (c / kDecStages) & 1, err, 0x34);
    }
    return;
  }

  // ---------------- consumers
  const int kw = lane >> 2;   // key of this lane within the warp's 8 keys
  const int q4 = lane & 3;    // quarter of the head dims this lane scores
  // chunk rotation: with it the 8 lanes of a quarter-warp read 8 different banks
  const int rot = QC == 4 ? (((kw & 1) << 1) | (q4 >> 1)) : (kw & 1);
  float qr[Q_IN_REGS ? NREP : 1][Q_IN_REGS ? QD : 1];
  if constexpr (Q_IN_REGS) {
#pragma unroll
    for (int r = 0; r < NREP; ++r)
#pragma unroll
      for (int i = 0; i < QC; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e)
          qr[r][i * 8 + e] = qs[r * DH + q4 * QD + ((i + rot) & (QC - 1)) * 8 + e];
  }
  float m_run[NREP], l_run[NREP], o[NREP][VD];
#pragma unroll
  for (int r = 0; r < NREP; ++r) {
    m_run[r] = -INFINITY;
    l_run[r] = 0.f;
#pragma unroll
    for (int j = 0; j < VD; ++j) o[r][j] = 0.f;
  }

  for (int c = 0; c < nch; ++c) {
    const int st = c % kDecStages;
    // warp-uniform: the lanes of a warp meet in full-mask shuffles below
    if (!mbar_wait_warp(&full[st], (c / kDecStages) & 1, err, 0x35)) break;
    const bf16* Ks = sKV + (2 * st) * (CHUNK_BYTES / 2);
    const bf16* Vs = sKV + (2 * st + 1) * (CHUNK_BYTES / 2);
    const int rows = min(kDecChunk, nk - c * kDecChunk);
    const int key = warp * 8 + kw;  // within the chunk
    const bool valid = key < rows;
    float s[NREP];
#pragma unroll
    for (int r = 0; r < NREP; ++r) s[r] = 0.f;
    if (valid) {
      const bf16* krow = Ks + key * DH + q4 * QD;
#pragma unroll
      for (int i = 0; i < QC; ++i) {
        const int ci = (i + rot) & (QC - 1);
        float kv8[8];
        load8(krow + ci * 8, kv8);
#pragma unroll
        for (int r = 0; r < NREP; ++r) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float qv = Q_IN_REGS ? qr[Q_IN_REGS ? r : 0][Q_IN_REGS ? i * 8 + e : 0]
                                       : qs[r * DH + q4 * QD + ci * 8 + e];
            s[r] = fmaf(qv, kv8[e], s[r]);
          }
        }
      }
    }
    // full dot product: sum the four quarters of each key
#pragma unroll
    for (int r = 0; r < NREP; ++r) {
      s[r] += __shfl_xor_sync(0xffffffffu, s[r], 1);
      s[r] += __shfl_xor_sync(0xffffffffu, s[r], 2);
      if (!valid) s[r] = -INFINITY;
    }
    // warp-level online softmax over the warp's keys of this chunk
    float p[NREP];
#pragma unroll
    for (int r = 0; r < NREP; ++r) {
      float mx = s[r];
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m_run[r], mx);
      // a warp may have seen no valid key yet (m_new = -inf): keep its state at zero
      const float alpha = m_new == -INFINITY ? 1.f : ex2_approx(m_run[r] - m_new);
      p[r] = valid ? ex2_approx(s[r] - m_new) : 0.f;
      float ps = p[r];
      ps += __shfl_xor_sync(0xffffffffu, ps, 4);
      ps += __shfl_xor_sync(0xffffffffu, ps, 8);
      ps += __shfl_xor_sync(0xffffffffu, ps, 16);
      l_run[r] = l_run[r] * alpha + ps;
      m_run[r] = m_new;
#pragma unroll
      for (int j = 0; j < VD; ++j) o[r][j] *= alpha;
    }
    // P V: lane owns dims [VD*lane, VD*lane + VD)
    const int nvalid = min(8, rows - warp * 8);  // warp-uniform
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      if (kk < nvalid) {
        const bf16* vrow = Vs + (warp * 8 + kk) * DH + lane * VD;
        float vv[VD];
        if constexpr (VD == 4) {
          const uint2 u = *reinterpret_cast<const uint2*>(vrow);
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
          const float2 bb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
          vv[0] = a.x; vv[1] = a.y; vv[2] = bb.x; vv[3] = bb.y;
        } else {
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vrow));
          vv[0] = a.x; vv[1] = a.y;
        }
#pragma unroll
        for (int r = 0; r < NREP; ++r) {
          const float pk = __shfl_sync(0xffffffffu, p[r], kk * 4);
#pragma unroll
          for (int j = 0; j < VD; ++j) o[r][j] = fmaf(pk, vv[j], o[r][j]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---------------- merge the 8 warps' states (the ring is free now)
  asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32) : "memory");
  float* mrg = reinterpret_cast<float*>(smem);  // [warp][NREP][DH + 2]
  constexpr int W = DH + 2;
#pragma unroll
  for (int r = 0; r < NREP; ++r) {
    float* dst = mrg + (warp * NREP + r) * W;
#pragma unroll
    for (int j = 0; j < VD; ++j) dst[lane * VD + j] = o[r][j];
    if (lane == 0) {
      dst[DH] = m_run[r];
      dst[DH + 1] = l_run[r];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32) : "memory");
  for (int e = threadIdx.x; e < NREP * DH; e += kDecWarps * 32) {
    const int r = e / DH, d = e % DH;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, mrg[(w * NREP + r) * W + DH]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float* src = mrg + (w * NREP + r) * W;
      const float wt = src[DH] == -INFINITY ? 0.f : ex2_approx(src[DH] - M);
      L += src[DH + 1] * wt;
      acc += src[d] * wt;
    }
    float* dst = out_base + r * head_stride;
    dst[d] = acc;
    if (d == 0) {
      dst[DH] = M;
      dst[DH + 1] = L;
    }
  }
}

// Merge the splits of one (b, h): M = max_s m_s, l = sum_s l_s 2^(m_s - M),
// o = sum_s o_s 2^(m_s - M) / l.
template <int DH>
__global__ void attn_decode_combine_kernel(const float* __restrict__ part, bf16* __restrict__ o,
                                           int H, int n_splits, const int* __restrict__ kv_len) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const int used = min(n_splits, (kv_len[b] + 1 + kDecSplitKeys - 1) / kDecSplitKeys);
  if (used <= 0) {  // negative length: the split kernel latched an error; write zeros
    o[((long long)b * H + h) * DH + d] = __float2bfloat16_rn(0.f);
    return;
  }
  const float* base = part + ((long long)b * H + h) * n_splits * (DH + 2);
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

template <int DH, int NREP>
static cudaError_t run_split(dim3 grid, const void* q, const void* k, const void* v, float* part,
                             int H, int Hkv, int k_stride, int n_splits, const int* kv_len,
                             float scale_log2, int* err, cudaStream_t s) {
  constexpr int smem = dec_smem_bytes<DH>(NREP);
  auto kern = attn_decode_split_kernel<DH, NREP>;
  static std::atomic<unsigned long long> attr_done{0};
  if (cudaError_t e = ensure_smem_attr(kern, smem, attr_done); e != cudaSuccess)
    return e;
  return launch_k(kern, grid, kDecThreads, smem, s, (const bf16*)q, (const bf16*)k, (const bf16*)v,
                  part, H, Hkv, k_stride, n_splits, kv_len, scale_log2, err);
}

template <int DH>
static cudaError_t run_decode(const void* q, const void* k, const void* v, void* o, float* part,
                              int B, int H, int Hkv, int k_stride, const int* kv_len, int* err,
                              cudaStream_t s) {
  const int n_splits = decode_attn_chunks(k_stride);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  const int g = decode_attn_heads_per_cta(H / Hkv);
  const dim3 grid(n_splits, H / g, B);
  cudaError_t e;
  switch (g) {
    case 1: e = run_split<DH, 1>(grid, q, k, v, part, H, Hkv, k_stride, n_splits, kv_len, scale_log2, err, s); break;
    case 2: e = run_split<DH, 2>(grid, q, k, v, part, H, Hkv, k_stride, n_splits, kv_len, scale_log2, err, s); break;
    case 4: e = run_split<DH, 4>(grid, q, k, v, part, H, Hkv, k_stride, n_splits, kv_len, scale_log2, err, s); break;
    default: e = run_split<DH, 8>(grid, q, k, v, part, H, Hkv, k_stride, n_splits, kv_len, scale_log2, err, s); break;
  }
  if (e != cudaSuccess) return e;
  return launch_k(attn_decode_combine_kernel<DH>, dim3(H, B), DH, 0, s, (const float*)part,
                  (bf16*)o, H, n_splits, kv_len);
}

cudaError_t launch_attn_decode(const void* q, const void* k, const void* v, void* o, float* part,
                               int B, int H, int Hkv, int dh, int k_stride, const int* kv_len,
                               int* err, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  if (Hkv <= 0 || H % Hkv) return cudaErrorInvalidValue;
  if (dh == 128) return run_decode<128>(q, k, v, o, part, B, H, Hkv, k_stride, kv_len, err, s);
  if (dh == 64) return run_decode<64>(q, k, v, o, part, B, H, Hkv, k_stride, kv_len, err, s);
  return cudaErrorInvalidValue;
}

}  // namespace lb
