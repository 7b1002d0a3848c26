// internal.h — launch interface between the C-ABI layer (capi.cu) and the kernels.
// Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

namespace lb {

enum { kF32 = 0, kBF16 = 1 };

// Codes latched into a device error word (first error wins).
enum : int {
  kErrNone = 0,
  kErrWaitBase = 0x100,     // + wait-site id: a bounded wait ran out
  kErrCacheBounds = 0x200,  // a KV-cache index outside [0, t_max)
  kErrPosBounds = 0x201,    // a RoPE position outside the table
};

// Split-K count actually used for K and a requested count: every split non-empty.
inline int gemm_effective_split(int K, int n_split) {
  const int KB = (K + 63) / 64;
  n_split = std::max(1, std::min(n_split, KB));
  const int per = (KB + n_split - 1) / n_split;
  return (KB + per - 1) / per;
}

// Raise `kern`'s dynamic shared-memory limit to `bytes` once per device: the attribute
// is per device and a process may drive several GPUs. `done` (one static per kernel)
// holds a bit per device ordinal < 64; larger ordinals set the attribute every time.
template <typename Kern>
inline cudaError_t ensure_smem_attr(Kern kern, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Launch `kern` on `s` with programmatic dependent launch allowed: the grid may
// start while the previous kernel on the stream finishes. Every kernel of this
// library executes griddepcontrol.wait (pdl_wait) before its first global-memory
// access, so only its prologue (barrier init, TMEM allocation, descriptor
// prefetch) overlaps the previous kernel.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Same, launched as clusters of two CTAs (a 2-SM MMA pair); grid.x must be even.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k_pair(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ----------------------------------------------------------- norm_fuse.cu
cudaError_t launch_resid_rmsnorm(int dtype, const void* x, const float* partial, int n_split,
                                 long long split_stride, void* x_out, const void* g, void* y,
                                 int rows, int d, float eps, cudaStream_t s);
cudaError_t launch_qkv_finish(int dtype, const float* qkv, int n_split, long long split_stride,
                              int M, int T, int H, int Hkv, int dh, const int* pos_base, int pos0,
                              const float* cos_t, const float* sin_t, int max_pos, void* q_out,
                              void* k_cache, void* v_cache, int t_max, int* err, cudaStream_t s);
cudaError_t launch_silu_mul(int dtype, const float* gu, int n_split, long long split_stride, int M,
                            int f, int n_packed, int block, void* a, cudaStream_t s);
// out = a + b per row of d (d % 8 == 0), with each stored row's sum of squares in ss_out
// when it is not NULL.
cudaError_t launch_add_rows(int dtype, const void* a, const void* b, void* out, float* ss_out,
                            int rows, int d, cudaStream_t s);
cudaError_t launch_resid_add(int dtype, const void* resid, const float* part, int n_split,
                             long long split_stride, void* out, long long total, int* lens, int B,
                             int len_inc, cudaStream_t s);
cudaError_t launch_set_lens(int* lens, int B, int value, cudaStream_t s);
// cos_t / sin_t rows [p0, p1) (each `half` = dh/2 wide) for rotary base `base`, in fp64.
cudaError_t launch_rope_table(float* cos_t, float* sin_t, int p0, int p1, int half, double base,
                              int dh, cudaStream_t s);
// ss[m] = sum_j x[m][j]^2 (fp32) for bf16 rows; zeroes ss_zero[m] (when given) for a
// later accumulation; block 0 also sets lens[0..B) = len_value (when lens given).
cudaError_t launch_row_ssq(const void* x, float* ss, float* ss_zero, int rows, int d, int* lens,
                           int B, int len_value, int* err, cudaStream_t s);
// w[r][c] = bf16(w[r][c] * g[c]) in place (bf16 [rows, cols], g [cols]).
cudaError_t launch_scale_cols(void* w, const void* g, long long rows, int cols, cudaStream_t s);
cudaError_t launch_rope_apply(int dtype, void* x, const int* pos, int B, int T, int H, int dh,
                              double base, cudaStream_t s);
cudaError_t launch_selftest_timeout(int* err, unsigned long long budget_ns, cudaStream_t s);

// ----------------------------------------------------------- simt_f32.cu (fp32 path)
// C[M,N] = A[M,K] B[N,K]^T (+ resid[M,N]); all fp32 row-major.
cudaError_t launch_gemm_f32(const float* A, const float* B, float* C, const float* resid, int M,
                            int N, int K, cudaStream_t s);
// Causal attention, fp32. q [B,H,Tq,dh]; k,v [B,Hkv,k_stride,dh]; o [B,Tq,H*dh].
// kv_len NULL: Tk keys, query i at Tk-Tq+i. kv_len[b] given: Tk_b = kv_len[b] + 1.
cudaError_t launch_attn_f32(const float* q, const float* k, const float* v, float* o, int B,
                            int Tq, int Tk, int H, int Hkv, int dh, int k_stride,
                            const int* kv_len, cudaStream_t s);

// ----------------------------------------------------------- gemm_tc.cu (bf16 tcgen05)
enum EpiKind {
  kEpiStore = 0,     // out[m][n] = bf16(acc)
  kEpiResid = 1,     // out[m][n] = bf16(resid[m][n] + acc)
  kEpiSwiGLU = 2,    // tile = [gate 128 | up 128] -> a[m][nt*128 + j] = bf16(silu(g)*u)
  kEpiQkvRope = 3,   // RoPE on Q/K heads, scatter Q to [B,H,T,dh], K/V into the cache
  kEpiPartialT = 4,  // swap-AB split-K: part[split][col][row] = acc (fp32)
};

struct GemmEpi {
  int kind = kEpiStore;
  void* out = nullptr;          // bf16 output / partial fp32 buffer
  const void* resid = nullptr;  // bf16 residual [M, N]
  long long ldo = 0;            // row stride of out / resid (elements)
  long long split_stride = 0;   // kEpiPartialT: elements between split slabs
  // kEpiQkvRope
  int f = 0;                    // kEpiSwiGLU: number of output columns (intermediate size)
  int T = 1, H = 0, Hkv = 0, dh = 128, t_max = 0, max_pos = 0;
  int pos0 = 0;  // kEpiQkvRope: position of token 0 (the cache length before the call)
  void* q_out = nullptr;
  void* k_cache = nullptr;
  void* v_cache = nullptr;
  const float* cos_t = nullptr;
  const float* sin_t = nullptr;
  int* err = nullptr;
  // RMSNorm folded into the GEMM (the gain is folded into the weights): when
  // row_ss != NULL the accumulator of row m is multiplied by
  // rsqrt(row_ss[m] * row_inv_d + row_eps) before the epilogue op (QkvRope, SwiGLU).
  const float* row_ss = nullptr;
  float row_inv_d = 0.f, row_eps = 0.f;
  // kEpiResid: when ss_out != NULL, the sum of squares of each stored (rounded)
  // output row is accumulated into ss_out[m] (atomically, over the N tiles).
  float* ss_out = nullptr;
  // Neither operand is written by the kernel launched just before this GEMM (which
  // triggered its dependents only after its own wait, so everything earlier is complete):
  // the TMA producer and the MMA issuer then start without waiting for that kernel; only
  // the epilogue does (it reads row_ss).
  bool operands_ready = false;
};

// D[M,N] = A[M,K] · B[N,K]^T, bf16 operands (K-major, row stride K), fp32 accumulation in
// TMEM. BN selects the N tile (256 / 128 / 32). n_split > 1 splits K (kEpiPartialT only).
cudaError_t launch_gemm_tc(const void* A, const void* B, int M, int N, int K, int BN, int n_split,
                           const GemmEpi& epi, int num_sms, cudaStream_t s);

// ----------------------------------------------------------- gemm_w8.cu (INT8 weights, decode)
// Depth (K elements) of one pipeline step of the INT8 decode GEMM, and of one tile of
// the blocked INT8 layout.
constexpr int kW8K = 128;
// INT8 codes are stored tile-blocked so that a decode GEMM streams each 128 x kW8K tile
// as one contiguous run: [ceil(rows/128)][ceil(cols/kW8K)] tiles (rows and cols padded
// with zero codes), each tile [kW8K/32 K quarters][128 rows][32].
__host__ __device__ inline long long w8_blocked_offset(int row, int col, int cols) {
  const long long tile = (long long)(row >> 7) * ((cols + kW8K - 1) / kW8K) + col / kW8K;
  return tile * (128 * kW8K) + ((col % kW8K) >> 5) * 4096 + (row & 127) * 32 + (col & 31);
}
inline size_t w8_blocked_bytes(int rows, int cols) {
  return (size_t)((rows + 127) / 128) * 128 * (size_t)((cols + kW8K - 1) / kW8K) * kW8K;
}
// Split-K slices of an INT8 decode GEMM over K (in kW8K-deep blocks) for a requested split.
inline int w8_effective_split(int K, int n_split) {
  const int KT = (K + kW8K - 1) / kW8K;
  n_split = std::max(1, std::min(n_split, KT));
  const int per = (KT + n_split - 1) / n_split;
  return (KT + per - 1) / per;
}
// q = rint(w / s_r), s_r = max_c |w[r][c]| / 127 (fp32), bf16 w [rows, cols] -> blocked q
// (zeroed beforehand by the caller), scale[rows].
cudaError_t launch_quantize_rows_int8(const void* w, void* q, float* scale, int rows, int cols,
                                      cudaStream_t s);
// Swap-AB decode GEMM with blocked INT8 weights A8 (M rows, row scales row_scale[M]) and
// bf16 tokens B [N <= 32, K]: part[split][token][row] = row_scale[row] * sum_k A8 B
// (kEpiPartialT layout), w8_effective_split(K, n_split) slices. K % 64 == 0.
cudaError_t launch_gemm_w8(const void* A8, const float* row_scale, const void* B, int M, int N,
                           int K, int n_split, const GemmEpi& epi, int num_sms, cudaStream_t s);

// ----------------------------------------------------------- attn_tc.cu (bf16 tcgen05)
// Causal flash attention. q [B,H,Tq,dh]; k,v [B,Hkv,k_stride,dh]; o [B,Tq,H*dh].
cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* o, int B, int Tq,
                           int Tk, int H, int Hkv, int dh, int k_stride, int* err,
                           cudaStream_t s);

// ----------------------------------------------------------- attn_decode.cu (bf16)
// Split-KV decode attention: one query per (b, h) at position kv_len[b], keys
// 0..kv_len[b] (the new key already appended). q [B,H,dh]; k,v [B,Hkv,k_stride,dh];
// o [B, H*dh]. `part` holds B*H*max_chunks*(dh+2) floats.
int decode_attn_chunks(int k_stride);
// Query heads one decode-attention CTA serves: the largest of 8, 4, 2, 1 dividing n_rep.
int decode_attn_heads_per_cta(int n_rep);
cudaError_t launch_attn_decode(const void* q, const void* k, const void* v, void* o, float* part,
                               int B, int H, int Hkv, int dh, int k_stride, const int* kv_len,
                               int* err, cudaStream_t s);

// ----------------------------------------------------------- tensor maps
// Encode a 2D bf16 tensor map over a row-major [rows, cols] matrix with a
// box of [box_rows, 64 cols] and 128-byte swizzle.
bool make_tmap_2d_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows);
// 3D bf16 tensor map over [planes, rows, cols] (cols contiguous, rows `cols` apart,
// planes `plane_stride` elements apart), box [1, box_rows, 64], 128-byte swizzle.
// Rows >= `rows` read as zero.
bool make_tmap_3d_bf16(CUtensorMap* m, const void* base, uint64_t planes, uint64_t rows,
                       uint64_t cols, uint64_t plane_stride, uint32_t box_rows);

}  // namespace lb
