// capi.cu — the C ABI of the library (include/llama_block.h): handle lifecycle,
// weight packing, RoPE table, workspace, and the launch sequences of prefill and
// decode. Host code only; every step of the block runs in the kernels of the
// other translation units.
//
// Prefill of the pre-norm layer (LMDrive page §2.5), bf16:
//   rmsnorm(X) -> h | tcgen05 GEMM h·Wqkv^T with RoPE + Q/K/V scatter | tcgen05 flash
//   attention -> O | GEMM O·Wo^T + X -> X' | rmsnorm(X') -> h2 |
//   GEMM h2·Wgu^T with SiLU(g)*u -> A | GEMM A·Wd^T + X' -> X''.
// Decode (chapter 04 of the mechanics page), bf16, B tokens: the same stages with
// swap-AB split-K tcgen05 GEMMs (weights stream as the 128-row operand, the B
// tokens are the N side), fp32 partials reduced by the small fused kernels, and
// split-KV attention over the cache.
// fp32 handles run the same stages on the fp32 SIMT kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/llama_block.h"
#include "internal.h"

using namespace lb;

// ------------------------------------------------------------------ errors
static thread_local std::string g_last_error = "no error";

static lb_status fail(lb_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

#define LB_CUDA(call)                                                                     \
  do {                                                                                    \
    cudaError_t e_ = (call);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return fail(e_ == cudaErrorMemoryAllocation ? LB_ERR_OOM : LB_ERR_CUDA, "%s: %s (%s:%d)", \
                  #call, cudaGetErrorString(e_), __FILE__, __LINE__);                     \
  } while (0)

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

namespace lb {

bool make_tmap_2d_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 15) || (cols * 2) % 16) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d_bf16(CUtensorMap* m, const void* base, uint64_t planes, uint64_t rows,
                       uint64_t cols, uint64_t plane_stride, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 15) || (cols * 2) % 16 ||
      (plane_stride * 2) % 16)
    return false;
  cuuint64_t dims[3] = {cols, rows, planes};
  cuuint64_t strides[2] = {cols * 2, plane_stride * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace lb

// ------------------------------------------------------------------ device info
static int num_sms_of_current_device() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// Error word of the standalone entry points, one per device.
// Makes the device a handle was created on current for the duration of a call (the
// caller's current device may differ), restoring the caller's afterwards.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (dev < 0) return;  // no handle: stay on the current device
    if (cudaGetDevice(&prev) != cudaSuccess) {
      prev = -1;
      ok = false;
    } else if (prev != dev && cudaSetDevice(dev) != cudaSuccess) {
      ok = false;
    }
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};
#define LB_ON_DEVICE(h, where)                                                   \
  DeviceGuard lb_device_guard((h)->device);                                      \
  if (!lb_device_guard.ok) return fail(LB_ERR_CUDA, "%s: cannot select the handle's device", where)

static std::mutex g_err_mu;
static std::map<int, int*> g_err_words;

// The standalone word of the current device if a call has created it (allocates nothing).
static int* existing_standalone_err_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  auto it = g_err_words.find(dev);
  return it == g_err_words.end() ? nullptr : it->second;
}

static int* standalone_err_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  auto it = g_err_words.find(dev);
  if (it != g_err_words.end()) return it->second;
  int* p = nullptr;
  if (cudaMalloc(&p, sizeof(int)) != cudaSuccess) return nullptr;
  if (cudaMemset(p, 0, sizeof(int)) != cudaSuccess) return nullptr;
  g_err_words[dev] = p;
  return p;
}

// ------------------------------------------------------------------ handle
struct llama_block {
  int d, H, Hkv, dh, f, max_pos, dtype, device, num_sms;
  float eps, base;
  size_t esz;
  int n_qkv;   // (H + 2 Hkv) * dh
  int f_pad;   // bf16: f rounded up to 128 (gate/up interleave block)
  int n_gu;    // rows of the packed gate/up weight
  void *w_qkv = nullptr, *w_o = nullptr, *w_gu = nullptr, *w_d = nullptr;
  void *g1 = nullptr, *g2 = nullptr;
  float *cos_t = nullptr, *sin_t = nullptr;
  // dynamic NTK RoPE scaling (llama_block_set_rope_dynamic_ntk): off when ntk_orig == 0;
  // rope_mixed: some table rows hold another base than `base`
  float ntk_factor = 1.f;
  int ntk_orig = 0;
  bool rope_mixed = false;
  int* err = nullptr;
  bool has_weights = false;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  std::vector<int> lens;  // host mirror of the cache lengths
  // INT8 decode weights (llama_block_quantize_decode_weights): codes and row scales of
  // the packed W_qkv, W_o, W_gu, W_d
  bool decode_int8 = false;
  void *q8[4] = {nullptr, nullptr, nullptr, nullptr};
  float* s8[4] = {nullptr, nullptr, nullptr, nullptr};
  // profiling: optional per-stage events, and the number of kernels launched
  bool timing = false;
  std::vector<cudaEvent_t> ev;            // 2 per stage
  std::vector<const char*> stage_names;   // stages of the last prefill/decode
  unsigned long long launches = 0;
};

static constexpr int kMaxStages = 16;

// Run one stage (one or more kernel launches) on stream s, bracketed by events
// when timing is enabled, and count its kernels.
#define LB_STAGE(name, nkern, call)                                                  \
  do {                                                                               \
    const int si_ = (int)b->stage_names.size();                                      \
    if (b->timing && si_ < kMaxStages) LB_CUDA(cudaEventRecord(b->ev[2 * si_], s));   \
    LB_CUDA(call);                                                                   \
    if (b->timing && si_ < kMaxStages) LB_CUDA(cudaEventRecord(b->ev[2 * si_ + 1], s)); \
    b->stage_names.push_back(name);                                                  \
    b->launches += (nkern);                                                          \
  } while (0)

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace carving: each region 256-byte aligned.
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base((char*)b) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off = align_up(off + bytes, 256);
    return p;
  }
};

struct PrefillWs {
  void *h, *q, *o, *x1, *a;
  float *qkv32, *gu32;
  float *ss1, *ss2;  // row sums of squares of X and X' (bf16 path)
};
struct DecodeWs {
  void *h, *q, *o, *x1, *a;
  float* part;
  float* attn_part;
};

// Split-K factor of a decode GEMM (m_tiles x n_tiles output tiles, K deep, tile_bytes
// streamed per 64-deep K block of a tile): the split whose busiest SM streams the
// fewest bytes -- whole waves of equal units over the SMs, a fixed cost per unit, and
// the fp32 partials (written, then read by the reduction) spread over all SMs.
static int decode_split(int m_tiles, int n_tiles, int bn, int K, int tile_bytes, int num_sms) {
  const int KB = (K + 63) / 64;
  const long long tiles = (long long)m_tiles * n_tiles;
  double best = 0;
  int best_s = 1;
  for (int sp = 1; sp <= std::min(KB, 64); ++sp) {
    const int per = (KB + sp - 1) / sp;
    if ((KB + per - 1) / per != sp) continue;  // the same units as a smaller split
    const long long units = tiles * sp;
    const long long waves = (units + num_sms - 1) / num_sms;
    const double cost = (double)waves * ((double)per * tile_bytes + 4096.0) +
                        (double)units * 128.0 * bn * 4 * 2 / num_sms;
    if (sp == 1 || cost < best * 0.999) {
      best = cost;
      best_s = sp;
    }
  }
  return best_s;
}

// Tile width and split of the four decode GEMMs (QKV, o_proj, gate/up, down) for a
// batch of B tokens, with the INT8 weights when w8 (used for B <= 32 only). split[i] is
// the number of partial slices the GEMM writes (canonical: no two splits give the same
// units), which the reducing kernel reads.
struct DecodePlan {
  int bn;
  bool w8;
  int split[4];
};

static DecodePlan decode_plan(const llama_block* b, int B, bool w8) {
  DecodePlan p;
  p.bn = B <= 32 ? 32 : B <= 64 ? 64 : B <= 128 ? 128 : 256;
  p.w8 = w8 && B <= 32;
  const int n_tiles = (B + p.bn - 1) / p.bn;
  const int M[4] = {b->n_qkv, b->d, b->n_gu, b->d};
  const int K[4] = {b->d, b->H * b->dh, b->d, b->f};
  for (int i = 0; i < 4; ++i) {
    if (p.w8)  // kW8K-deep K blocks of INT8 + the token tile
      p.split[i] = decode_split((M[i] + 127) / 128, n_tiles, p.bn, (K[i] + kW8K - 1) / kW8K * 64,
                                128 * kW8K + p.bn * kW8K * 2, b->num_sms);
    else
      p.split[i] = decode_split((M[i] + 127) / 128, n_tiles, p.bn, K[i], 128 * 64 * 2 + p.bn * 64 * 2,
                                b->num_sms);
  }
  return p;
}

static PrefillWs carve_prefill(const llama_block* b, void* base, int M, size_t* total) {
  Carver c(base);
  PrefillWs w;
  w.h = c.take((size_t)M * b->d * b->esz);
  w.q = c.take((size_t)M * b->H * b->dh * b->esz);
  w.o = c.take((size_t)M * b->H * b->dh * b->esz);
  w.x1 = c.take((size_t)M * b->d * b->esz);
  w.a = c.take((size_t)M * b->f_pad * b->esz);
  if (b->dtype == kF32) {
    w.qkv32 = (float*)c.take((size_t)M * b->n_qkv * 4);
    w.gu32 = (float*)c.take((size_t)M * b->n_gu * 4);
    w.ss1 = w.ss2 = nullptr;
  } else {
    w.qkv32 = w.gu32 = nullptr;
    w.ss1 = (float*)c.take((size_t)M * 4);
    w.ss2 = (float*)c.take((size_t)M * 4);
  }
  *total = c.off;
  return w;
}

static DecodeWs carve_decode(const llama_block* b, void* base, int B, int t_max, size_t* total) {
  Carver c(base);
  DecodeWs w;
  w.h = c.take((size_t)B * b->d * b->esz);
  w.q = c.take((size_t)B * b->H * b->dh * b->esz);
  w.o = c.take((size_t)B * b->H * b->dh * b->esz);
  w.x1 = c.take((size_t)B * b->d * b->esz);
  w.a = c.take((size_t)B * b->f_pad * b->esz);
  size_t part = 0;
  if (b->dtype == kBF16) {
    // room for the partials of every batch size up to B, bf16 or INT8 weights, so that
    // a workspace reserved for B is never regrown by a smaller decode
    const size_t M[4] = {(size_t)b->n_qkv, (size_t)b->d, (size_t)b->n_gu, (size_t)b->d};
    for (int bb = 1; bb <= B; ++bb)
      for (int w8 = 0; w8 < 2; ++w8) {
        const DecodePlan p = decode_plan(b, bb, w8 != 0);
        for (int i = 0; i < 4; ++i) part = std::max(part, (size_t)p.split[i] * bb * M[i]);
      }
  } else {
    part = std::max((size_t)B * b->n_qkv, (size_t)B * b->n_gu);
  }
  w.part = (float*)c.take(part * 4);
  w.attn_part = (float*)c.take((size_t)B * b->H * decode_attn_chunks(t_max) * (b->dh + 2) * 4);
  *total = c.off;
  return w;
}

static lb_status ensure_ws(llama_block* b, size_t need) {
  if (need <= b->ws_bytes) return LB_OK;
  if (b->ws) {
    LB_CUDA(cudaDeviceSynchronize());
    LB_CUDA(cudaFree(b->ws));
    b->ws = nullptr;
    b->ws_bytes = 0;
  }
  LB_CUDA(cudaMalloc(&b->ws, need));
  b->ws_bytes = need;
  return LB_OK;
}

extern "C" {

const char* llama_block_last_error(void) { return g_last_error.c_str(); }

size_t llama_block_kv_cache_bytes(int B, int n_kv_heads, int head_dim, int t_max, lb_dtype dtype) {
  if (B <= 0 || n_kv_heads <= 0 || head_dim <= 0 || t_max <= 0) return 0;
  if (dtype != LB_F32 && dtype != LB_BF16) return 0;
  const size_t es = dtype == LB_F32 ? 4 : 2;
  return (size_t)2 * B * t_max * n_kv_heads * head_dim * es;
}

lb_status llama_block_create(int d, int n_heads, int n_kv_heads, int head_dim, int f, float eps,
                             float rope_base, lb_dtype dtype, int max_pos, llama_block** out) {
  if (!out) return fail(LB_ERR_INVALID_ARG, "create: out is NULL");
  *out = nullptr;
  if (d <= 0 || n_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || f <= 0 || max_pos <= 0)
    return fail(LB_ERR_INVALID_ARG, "create: sizes must be positive");
  if (!(eps > 0.f) || !(rope_base > 0.f))
    return fail(LB_ERR_INVALID_ARG, "create: eps and rope_base must be positive");
  if (dtype != LB_F32 && dtype != LB_BF16) return fail(LB_ERR_INVALID_ARG, "create: bad dtype");
  if (head_dim != 64 && head_dim != 128)
    return fail(LB_ERR_UNSUPPORTED, "create: head_dim %d not in {64,128}", head_dim);
  if (n_heads % n_kv_heads != 0)
    return fail(LB_ERR_UNSUPPORTED, "create: n_heads %% n_kv_heads != 0");
  if (d % 8 != 0 || d > 8192)
    return fail(LB_ERR_UNSUPPORTED, "create: d must be a multiple of 8 and <= 8192");
  if (dtype == LB_BF16 && (d % 64 != 0 || f % 8 != 0 || (n_heads * head_dim) % 64 != 0))
    return fail(LB_ERR_UNSUPPORTED, "create: bf16 needs d %% 64 == 0 and f %% 8 == 0");

  llama_block* b = new llama_block();
  b->d = d;
  b->H = n_heads;
  b->Hkv = n_kv_heads;
  b->dh = head_dim;
  b->f = f;
  b->max_pos = max_pos;
  b->dtype = dtype;
  b->eps = eps;
  b->base = rope_base;
  b->esz = dtype == LB_F32 ? 4 : 2;
  b->n_qkv = (n_heads + 2 * n_kv_heads) * head_dim;
  b->f_pad = dtype == LB_BF16 ? (f + 127) / 128 * 128 : f;
  b->n_gu = 2 * b->f_pad;

  auto cleanup_fail = [&](lb_status st) {
    llama_block_destroy(b);
    return st;
  };
  if (cudaGetDevice(&b->device) != cudaSuccess) {
    cudaGetLastError();
    delete b;
    return fail(LB_ERR_CUDA, "create: no CUDA device");
  }
  b->num_sms = num_sms_of_current_device();
  const size_t es = b->esz;
  if (cudaMalloc(&b->w_qkv, (size_t)b->n_qkv * d * es) != cudaSuccess ||
      cudaMalloc(&b->w_o, (size_t)d * n_heads * head_dim * es) != cudaSuccess ||
      cudaMalloc(&b->w_gu, (size_t)b->n_gu * d * es) != cudaSuccess ||
      cudaMalloc(&b->w_d, (size_t)d * f * es) != cudaSuccess ||
      cudaMalloc(&b->g1, (size_t)d * es) != cudaSuccess ||
      cudaMalloc(&b->g2, (size_t)d * es) != cudaSuccess ||
      cudaMalloc(&b->cos_t, (size_t)max_pos * (head_dim / 2) * 4) != cudaSuccess ||
      cudaMalloc(&b->sin_t, (size_t)max_pos * (head_dim / 2) * 4) != cudaSuccess ||
      cudaMalloc(&b->err, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    fail(LB_ERR_OOM, "create: device allocation failed");
    return cleanup_fail(LB_ERR_OOM);
  }
  // RoPE table (LMDrive page §2.2): inv_freq_i = base^(-2i/dh), angle = pos * inv_freq_i,
  // formed in fp64 on the host and stored as fp32 cos / sin [max_pos][dh/2].
  const int half = head_dim / 2;
  std::vector<float> ct((size_t)max_pos * half), st((size_t)max_pos * half);
  for (int i = 0; i < half; ++i) {
    const double inv = 1.0 / std::pow((double)rope_base, (2.0 * i) / (double)head_dim);
    for (int p = 0; p < max_pos; ++p) {
      const double a = (double)p * inv;
      ct[(size_t)p * half + i] = (float)std::cos(a);
      st[(size_t)p * half + i] = (float)std::sin(a);
    }
  }
  if (cudaMemcpy(b->cos_t, ct.data(), ct.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(b->sin_t, st.data(), st.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemset(b->err, 0, sizeof(int)) != cudaSuccess ||
      cudaMemset(b->w_gu, 0, (size_t)b->n_gu * d * es) != cudaSuccess) {
    cudaGetLastError();
    fail(LB_ERR_CUDA, "create: device initialisation failed");
    return cleanup_fail(LB_ERR_CUDA);
  }
  *out = b;
  return LB_OK;
}

void llama_block_destroy(llama_block* b) {
  if (!b) return;
  DeviceGuard dg(b->device);
  cudaDeviceSynchronize();
  for (cudaEvent_t e : b->ev) cudaEventDestroy(e);
  for (void* p : {b->w_qkv, b->w_o, b->w_gu, b->w_d, b->g1, b->g2, (void*)b->cos_t,
                  (void*)b->sin_t, (void*)b->err, b->ws})
    if (p) cudaFree(p);
  for (int i = 0; i < 4; ++i) {
    if (b->q8[i]) cudaFree(b->q8[i]);
    if (b->s8[i]) cudaFree(b->s8[i]);
  }
  delete b;
}

// Rows and columns of the four packed weight matrices (Q|K|V, o_proj, gate/up, down).
static void packed_shapes(const llama_block* b, int rows[4], int cols[4]) {
  rows[0] = b->n_qkv;  cols[0] = b->d;
  rows[1] = b->d;      cols[1] = b->H * b->dh;
  rows[2] = b->n_gu;   cols[2] = b->d;
  rows[3] = b->d;      cols[3] = b->f;
}

static lb_status quantize_packed(llama_block* b, cudaStream_t s) {
  int rows[4], cols[4];
  packed_shapes(b, rows, cols);
  void* w[4] = {b->w_qkv, b->w_o, b->w_gu, b->w_d};
  for (int i = 0; i < 4; ++i) {
    const size_t qbytes = w8_blocked_bytes(rows[i], cols[i]);
    if (!b->q8[i]) LB_CUDA(cudaMalloc(&b->q8[i], qbytes));
    if (!b->s8[i]) LB_CUDA(cudaMalloc(&b->s8[i], (size_t)rows[i] * sizeof(float)));
    LB_CUDA(cudaMemsetAsync(b->q8[i], 0, qbytes, s));  // the padding rows of the last tile
    LB_CUDA(launch_quantize_rows_int8(w[i], b->q8[i], b->s8[i], rows[i], cols[i], s));
  }
  return LB_OK;
}

lb_status llama_block_set_weights(llama_block* b, const void* wq, const void* wk, const void* wv,
                                  const void* wo, const void* w_gate, const void* w_up,
                                  const void* w_down, const void* g_attn, const void* g_mlp,
                                  void* stream) {
  if (!b) return fail(LB_ERR_INVALID_ARG, "set_weights: NULL handle");
  LB_ON_DEVICE(b, "set_weights");
  if (!wq || !wk || !wv || !wo || !w_gate || !w_up || !w_down || !g_attn || !g_mlp)
    return fail(LB_ERR_INVALID_ARG, "set_weights: NULL weight pointer");
  cudaStream_t s = (cudaStream_t)stream;
  const size_t es = b->esz, d = b->d;
  const size_t nq = (size_t)b->H * b->dh, nkv = (size_t)b->Hkv * b->dh;
  char* qkv = (char*)b->w_qkv;
  // fused Q | K | V rows
  LB_CUDA(cudaMemcpyAsync(qkv, wq, nq * d * es, cudaMemcpyDeviceToDevice, s));
  LB_CUDA(cudaMemcpyAsync(qkv + nq * d * es, wk, nkv * d * es, cudaMemcpyDeviceToDevice, s));
  LB_CUDA(cudaMemcpyAsync(qkv + (nq + nkv) * d * es, wv, nkv * d * es, cudaMemcpyDeviceToDevice, s));
  LB_CUDA(cudaMemcpyAsync(b->w_o, wo, d * nq * es, cudaMemcpyDeviceToDevice, s));
  LB_CUDA(cudaMemcpyAsync(b->w_d, w_down, d * b->f * es, cudaMemcpyDeviceToDevice, s));
  LB_CUDA(cudaMemcpyAsync(b->g1, g_attn, d * es, cudaMemcpyDeviceToDevice, s));
  LB_CUDA(cudaMemcpyAsync(b->g2, g_mlp, d * es, cudaMemcpyDeviceToDevice, s));
  char* gu = (char*)b->w_gu;
  if (b->dtype == kF32) {
    // [gate ; up]
    LB_CUDA(cudaMemcpyAsync(gu, w_gate, (size_t)b->f * d * es, cudaMemcpyDeviceToDevice, s));
    LB_CUDA(cudaMemcpyAsync(gu + (size_t)b->f * d * es, w_up, (size_t)b->f * d * es,
                            cudaMemcpyDeviceToDevice, s));
  } else {
    // blocks of 128 rows: [gate rows 128j.. | up rows 128j..] for j = 0, 1, ...
    const size_t blk = 128 * d * es;
    const int full_blocks = b->f / 128;
    if (full_blocks > 0) {
      LB_CUDA(cudaMemcpy2DAsync(gu, 2 * blk, w_gate, blk, blk, full_blocks,
                                cudaMemcpyDeviceToDevice, s));
      LB_CUDA(cudaMemcpy2DAsync(gu + blk, 2 * blk, w_up, blk, blk, full_blocks,
                                cudaMemcpyDeviceToDevice, s));
    }
    const int rem = b->f - full_blocks * 128;
    if (rem > 0) {
      const size_t src = (size_t)full_blocks * blk;
      LB_CUDA(cudaMemcpyAsync(gu + 2 * src, (const char*)w_gate + src, rem * d * es,
                              cudaMemcpyDeviceToDevice, s));
      LB_CUDA(cudaMemcpyAsync(gu + 2 * src + blk, (const char*)w_up + src, rem * d * es,
                              cudaMemcpyDeviceToDevice, s));
    }
  }
  if (b->dtype == kBF16) {
    // RMSNorm gains folded into the weights that read the normalised rows:
    // (g * x * r) W^T = r * x (W diag(g))^T; the GEMM epilogues apply r.
    LB_CUDA(launch_scale_cols(b->w_qkv, g_attn, b->n_qkv, b->d, s));
    LB_CUDA(launch_scale_cols(b->w_gu, g_mlp, b->n_gu, b->d, s));
  }
  b->has_weights = true;
  if (b->decode_int8) return quantize_packed(b, s);  // keep the INT8 copies in step
  return LB_OK;
}

lb_status llama_block_quantize_decode_weights(llama_block* b, int enable, void* stream) {
  if (!b) return fail(LB_ERR_INVALID_ARG, "quantize_decode_weights: NULL handle");
  LB_ON_DEVICE(b, "quantize_decode_weights");
  if (!enable) {
    LB_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
    for (int i = 0; i < 4; ++i) {
      if (b->q8[i]) LB_CUDA(cudaFree(b->q8[i]));
      if (b->s8[i]) LB_CUDA(cudaFree(b->s8[i]));
      b->q8[i] = nullptr;
      b->s8[i] = nullptr;
    }
    b->decode_int8 = false;
    return LB_OK;
  }
  if (b->dtype != kBF16)
    return fail(LB_ERR_UNSUPPORTED, "quantize_decode_weights: INT8 decode weights need LB_BF16");
  if (!b->has_weights) return fail(LB_ERR_NO_WEIGHTS, "quantize_decode_weights: set_weights first");
  int rows[4], cols[4];
  packed_shapes(b, rows, cols);
  for (int i = 0; i < 4; ++i)
    if (cols[i] % 64) return fail(LB_ERR_UNSUPPORTED, "quantize_decode_weights: K %% 64 != 0");
  const lb_status st = quantize_packed(b, (cudaStream_t)stream);
  if (st != LB_OK) return st;
  b->decode_int8 = true;
  return LB_OK;
}

lb_status llama_block_set_rope_dynamic_ntk(llama_block* b, float factor, int original_max_pos,
                                           void* stream) {
  if (!b) return fail(LB_ERR_INVALID_ARG, "set_rope_dynamic_ntk: NULL handle");
  LB_ON_DEVICE(b, "set_rope_dynamic_ntk");
  if (original_max_pos == 0) {  // off: plain RoPE everywhere again
    b->ntk_orig = 0;
    b->ntk_factor = 1.f;
    if (b->rope_mixed) {
      LB_CUDA(launch_rope_table(b->cos_t, b->sin_t, 0, b->max_pos, b->dh / 2, (double)b->base, b->dh,
                                (cudaStream_t)stream));
      b->rope_mixed = false;
    }
    return LB_OK;
  }
  if (original_max_pos < 0 || !(factor >= 1.f) || !std::isfinite(factor))
    return fail(LB_ERR_INVALID_ARG,
                "set_rope_dynamic_ntk: need factor >= 1 and original_max_pos > 0 (0 turns it off)");
  b->ntk_factor = factor;
  b->ntk_orig = original_max_pos;
  return LB_OK;
}

lb_status llama_block_reserve(llama_block* b, int max_tokens, int max_batch) {
  if (!b) return fail(LB_ERR_INVALID_ARG, "reserve: NULL handle");
  LB_ON_DEVICE(b, "reserve");
  if (max_tokens < 0 || max_batch < 0) return fail(LB_ERR_INVALID_ARG, "reserve: negative size");
  size_t a = 0, c = 0;
  carve_prefill(b, nullptr, max_tokens, &a);
  carve_decode(b, nullptr, max_batch, b->max_pos, &c);
  return ensure_ws(b, std::max(a, c));
}

lb_status llama_block_set_lengths(llama_block* b, const int32_t* lens_host, int B) {
  if (!b || !lens_host || B <= 0) return fail(LB_ERR_INVALID_ARG, "set_lengths: bad argument");
  b->lens.assign(lens_host, lens_host + B);
  return LB_OK;
}

// Dynamic NTK scaling (the rotary embedding of the LMDrive page §2.2 "supports dynamic
// NTK scaling to extend the maximum sequence length"; the pages give no formula, the
// reading taken is the dynamic NTK-aware rule): a call whose longest sequence reaches
// L > L0 tokens (L0 = the trained context) rotates its new tokens with
//   base' = base * (factor * L / L0 - (factor - 1)) ^ (dh / (dh - 2)),
// which leaves the highest frequency alone and stretches the lowest one's wavelength by
// exactly factor * L / L0 - (factor - 1); keys already in the cache keep their rotation.
static double call_rope_base(const llama_block* b, int L) {
  if (b->ntk_orig <= 0 || L <= b->ntk_orig) return (double)b->base;
  const double s = (double)b->ntk_factor * L / b->ntk_orig - ((double)b->ntk_factor - 1.0);
  return (double)b->base * std::pow(s, (double)b->dh / (double)(b->dh - 2));
}

// Whether a call reaching length L must first rewrite the table rows it reads.
static bool rope_rows_stale(const llama_block* b, int L) {
  return b->rope_mixed || call_rope_base(b, L) != (double)b->base;
}

// Rewrite table rows [p0, p1) for the base of a call reaching length L.
static cudaError_t update_rope_rows(llama_block* b, int p0, int p1, int L, cudaStream_t s) {
  const double base = call_rope_base(b, L);
  if (base != (double)b->base) b->rope_mixed = true;
  return launch_rope_table(b->cos_t, b->sin_t, p0, p1, b->dh / 2, base, b->dh, s);
}

static lb_status check_cache_args(llama_block* b, const void* x, const void* y, int B,
                                  const void* kc, const void* vc, int t_max, const int32_t* lens,
                                  const char* who) {
  if (!b) return fail(LB_ERR_INVALID_ARG, "%s: NULL handle", who);
  if (!x || !y || !kc || !vc || !lens) return fail(LB_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (B <= 0 || t_max <= 0) return fail(LB_ERR_INVALID_ARG, "%s: B and t_max must be positive", who);
  if (x == y) return fail(LB_ERR_INVALID_ARG, "%s: y must not alias x", who);
  if (!b->has_weights) return fail(LB_ERR_NO_WEIGHTS, "%s: set_weights was not called", who);
  return LB_OK;
}

// Prefill of T tokens per sequence appended at cache position L (L = 0: a fresh
// prefill; L > 0: chunked prefill into an existing cache).
static lb_status run_prefill(llama_block* b, const void* x, void* y, int B, int T, int L,
                             void* k_cache, void* v_cache, int t_max, int32_t* cache_len,
                             cudaStream_t s) {
  lb_status st;
  const int M = B * T;
  size_t need = 0;
  carve_prefill(b, nullptr, M, &need);
  if ((st = ensure_ws(b, need)) != LB_OK) return st;
  PrefillWs w = carve_prefill(b, b->ws, M, &need);
  const int d = b->d, H = b->H, Hkv = b->Hkv, dh = b->dh, f = b->f;

  b->stage_names.clear();
  if (rope_rows_stale(b, L + T))  // dynamic NTK: positions L .. L+T-1 for this call's base
    LB_STAGE("rope_table", 1, update_rope_rows(b, L, L + T, L + T, s));
  if (b->dtype == kBF16) {
    // RMSNorm statistics of X (its gain is folded into W_qkv); also zeroes the X'
    // statistic accumulated by o_proj and sets cache_len = L + T.
    LB_STAGE("row_stats_attn", 1, launch_row_ssq(x, w.ss1, w.ss2, M, d, cache_len, B, L + T, b->err, s));
    GemmEpi e1;
    e1.kind = kEpiQkvRope;
    e1.T = T; e1.H = H; e1.Hkv = Hkv; e1.dh = dh; e1.t_max = t_max; e1.max_pos = b->max_pos;
    e1.q_out = w.q; e1.k_cache = k_cache; e1.v_cache = v_cache; e1.pos0 = L;
    e1.cos_t = b->cos_t; e1.sin_t = b->sin_t; e1.err = b->err;
    e1.row_ss = w.ss1; e1.row_inv_d = 1.f / d; e1.row_eps = b->eps;
    e1.operands_ready = true;  // x and W_qkv: only the epilogue needs row_ssq's statistics
    LB_STAGE("qkv_rope_gemm", 1, launch_gemm_tc(x, b->w_qkv, M, b->n_qkv, d, 256, 1, e1, b->num_sms, s));
    LB_STAGE("attention", 1,
             launch_attn_tc(w.q, k_cache, v_cache, w.o, B, T, L + T, H, Hkv, dh, t_max, b->err, s));
    GemmEpi e2;
    e2.kind = kEpiResid; e2.out = w.x1; e2.resid = x; e2.ldo = d; e2.err = b->err;
    e2.ss_out = w.ss2;  // statistic of X' for the MLP's RMSNorm
    LB_STAGE("o_proj_resid_gemm", 1, launch_gemm_tc(w.o, b->w_o, M, d, H * dh, 256, 1, e2, b->num_sms, s));
    GemmEpi e3;
    e3.kind = kEpiSwiGLU; e3.out = w.a; e3.ldo = f; e3.f = f; e3.err = b->err;
    e3.row_ss = w.ss2; e3.row_inv_d = 1.f / d; e3.row_eps = b->eps;
    LB_STAGE("gate_up_swiglu_gemm", 1, launch_gemm_tc(w.x1, b->w_gu, M, b->n_gu, d, 256, 1, e3, b->num_sms, s));
    GemmEpi e4;
    e4.kind = kEpiResid; e4.out = y; e4.resid = w.x1; e4.ldo = d; e4.err = b->err;
    LB_STAGE("down_resid_gemm", 1, launch_gemm_tc(w.a, b->w_d, M, d, f, 256, 1, e4, b->num_sms, s));
  } else {
    const float* X = (const float*)x;
    LB_STAGE("rmsnorm_attn", 1,
             launch_resid_rmsnorm(kF32, x, nullptr, 0, 0, nullptr, b->g1, w.h, M, d, b->eps, s));
    LB_STAGE("qkv_gemm", 1, launch_gemm_f32((const float*)w.h, (const float*)b->w_qkv, w.qkv32, nullptr, M,
                                            b->n_qkv, d, s));
    LB_STAGE("qkv_rope", 1, launch_qkv_finish(kF32, w.qkv32, 1, 0, M, T, H, Hkv, dh, nullptr, L, b->cos_t,
                                              b->sin_t, b->max_pos, w.q, k_cache, v_cache, t_max,
                                              b->err, s));
    LB_STAGE("attention", 1, launch_attn_f32((const float*)w.q, (const float*)k_cache,
                                             (const float*)v_cache, (float*)w.o, B, T, L + T, H, Hkv,
                                             dh, t_max, nullptr, s));
    LB_STAGE("o_proj_resid_gemm", 1, launch_gemm_f32((const float*)w.o, (const float*)b->w_o,
                                                     (float*)w.x1, X, M, d, H * dh, s));
    LB_STAGE("rmsnorm_mlp", 1,
             launch_resid_rmsnorm(kF32, w.x1, nullptr, 0, 0, nullptr, b->g2, w.h, M, d, b->eps, s));
    LB_STAGE("gate_up_gemm", 1, launch_gemm_f32((const float*)w.h, (const float*)b->w_gu, w.gu32, nullptr,
                                                M, b->n_gu, d, s));
    LB_STAGE("silu_mul", 1, launch_silu_mul(kF32, w.gu32, 1, 0, M, f, b->n_gu, 0, w.a, s));
    LB_STAGE("down_resid_gemm", 1, launch_gemm_f32((const float*)w.a, (const float*)b->w_d, (float*)y,
                                                   (const float*)w.x1, M, d, f, s));
    LB_STAGE("set_lengths", 1, launch_set_lens(cache_len, B, L + T, s));
  }
  b->lens.assign(B, L + T);
  return LB_OK;
}

lb_status llama_block_prefill(llama_block* b, const void* x, void* y, int B, int T, void* k_cache,
                              void* v_cache, int t_max, int32_t* cache_len, void* stream) {
  lb_status st = check_cache_args(b, x, y, B, k_cache, v_cache, t_max, cache_len, "prefill");
  if (st != LB_OK) return st;
  LB_ON_DEVICE(b, "prefill");
  if (T <= 0) return fail(LB_ERR_INVALID_ARG, "prefill: T must be positive");
  if (T > t_max || T > b->max_pos)
    return fail(LB_ERR_CACHE_FULL, "prefill: T=%d exceeds t_max=%d or max_pos=%d", T, t_max,
                b->max_pos);
  return run_prefill(b, x, y, B, T, 0, k_cache, v_cache, t_max, cache_len, (cudaStream_t)stream);
}

lb_status llama_block_extend(llama_block* b, const void* x, void* y, int B, int T, void* k_cache,
                             void* v_cache, int t_max, int32_t* cache_len, void* stream) {
  lb_status st = check_cache_args(b, x, y, B, k_cache, v_cache, t_max, cache_len, "extend");
  if (st != LB_OK) return st;
  LB_ON_DEVICE(b, "extend");
  if (T <= 0) return fail(LB_ERR_INVALID_ARG, "extend: T must be positive");
  if ((int)b->lens.size() != B)
    return fail(LB_ERR_INVALID_ARG,
                "extend: the handle knows %d sequence lengths, B=%d (call prefill or set_lengths)",
                (int)b->lens.size(), B);
  const int L = b->lens[0];
  for (int i = 1; i < B; ++i)
    if (b->lens[i] != L)
      return fail(LB_ERR_UNSUPPORTED, "extend: the sequences have different cache lengths");
  if (L < 0 || L + T > t_max || L + T > b->max_pos)
    return fail(LB_ERR_CACHE_FULL, "extend: length %d + %d exceeds t_max=%d or max_pos=%d", L, T,
                t_max, b->max_pos);
  return run_prefill(b, x, y, B, T, L, k_cache, v_cache, t_max, cache_len, (cudaStream_t)stream);
}

lb_status llama_block_decode(llama_block* b, const void* x, void* y, int B, void* k_cache,
                             void* v_cache, int t_max, int32_t* cache_len, void* stream) {
  lb_status st = check_cache_args(b, x, y, B, k_cache, v_cache, t_max, cache_len, "decode");
  if (st != LB_OK) return st;
  LB_ON_DEVICE(b, "decode");
  if ((int)b->lens.size() != B)
    return fail(LB_ERR_INVALID_ARG,
                "decode: the handle knows %d sequence lengths, B=%d (call prefill or set_lengths)",
                (int)b->lens.size(), B);
  for (int i = 0; i < B; ++i)
    if (b->lens[i] < 0 || b->lens[i] + 1 > t_max || b->lens[i] >= b->max_pos)
      return fail(LB_ERR_CACHE_FULL, "decode: sequence %d at length %d cannot grow (t_max=%d, max_pos=%d)",
                  i, b->lens[i], t_max, b->max_pos);
  cudaStream_t s = (cudaStream_t)stream;
  size_t need = 0;
  carve_decode(b, nullptr, B, t_max, &need);
  if ((st = ensure_ws(b, need)) != LB_OK) return st;
  DecodeWs w = carve_decode(b, b->ws, B, t_max, &need);
  const int d = b->d, H = b->H, Hkv = b->Hkv, dh = b->dh, f = b->f;

  b->stage_names.clear();
  {  // dynamic NTK: the rows at the sequences' positions, for this step's base
    int lo = b->lens[0], hi = b->lens[0] + 1;
    for (int v : b->lens) {
      lo = std::min(lo, v);
      hi = std::max(hi, v + 1);
    }
    if (rope_rows_stale(b, hi)) LB_STAGE("rope_table", 1, update_rope_rows(b, lo, hi, hi, s));
  }
  if (b->dtype == kBF16) {
    const DecodePlan plan = decode_plan(b, B, b->decode_int8);
    const int bn = plan.bn;
    const bool w8 = plan.w8;
    // weight matrix i as the decode GEMM's 128-row operand: INT8 codes + row scales, or bf16
    auto wgemm = [&](int i, const void* wbf, const void* act, int Mw, int Kw, int split,
                     const GemmEpi& ep) -> cudaError_t {
      if (w8) return launch_gemm_w8(b->q8[i], b->s8[i], act, Mw, B, Kw, split, ep, b->num_sms, s);
      return launch_gemm_tc(wbf, act, Mw, B, Kw, bn, split, ep, b->num_sms, s);
    };
    // gains are folded into W_qkv / W_gu: the norms here only scale by 1/RMS
    LB_STAGE("rmsnorm_attn", 1,
             launch_resid_rmsnorm(kBF16, x, nullptr, 0, 0, nullptr, nullptr, w.h, B, d, b->eps, s));
    // Q|K|V: part[s][token][feature]
    GemmEpi e;
    e.kind = kEpiPartialT; e.out = w.part; e.err = b->err;
    e.ldo = b->n_qkv; e.split_stride = (long long)B * b->n_qkv;
    const int s1 = plan.split[0];
    LB_STAGE("qkv_gemm", 1, wgemm(0, b->w_qkv, w.h, b->n_qkv, d, s1, e));
    LB_STAGE("qkv_rope_append", 1,
             launch_qkv_finish(kBF16, w.part, s1, e.split_stride, B, 1, H,
                               Hkv, dh, cache_len, 0, b->cos_t, b->sin_t, b->max_pos, w.q, k_cache,
                               v_cache, t_max, b->err, s));
    LB_STAGE("attention", 2, launch_attn_decode(w.q, k_cache, v_cache, w.o, w.attn_part, B, H, Hkv,
                                                dh, t_max, cache_len, b->err, s));
    // o_proj, then X' = X + sum(partials) and h2 = RMSNorm(X') in one kernel
    const int K2 = H * dh;
    const int s2 = plan.split[1];
    e.ldo = d; e.split_stride = (long long)B * d;
    LB_STAGE("o_proj_gemm", 1, wgemm(1, b->w_o, w.o, d, K2, s2, e));
    LB_STAGE("resid_rmsnorm_mlp", 1,
             launch_resid_rmsnorm(kBF16, x, w.part, s2, e.split_stride,
                                  w.x1, nullptr, w.h, B, d, b->eps, s));
    // gate/up (packed rows), SiLU(g) * u
    const int s3 = plan.split[2];
    e.ldo = b->n_gu; e.split_stride = (long long)B * b->n_gu;
    LB_STAGE("gate_up_gemm", 1, wgemm(2, b->w_gu, w.h, b->n_gu, d, s3, e));
    LB_STAGE("silu_mul", 1, launch_silu_mul(kBF16, w.part, s3, e.split_stride,
                                            B, f, b->n_gu, 128, w.a, s));
    // down, y = X' + sum(partials); cache_len += 1
    const int s4 = plan.split[3];
    e.ldo = d; e.split_stride = (long long)B * d;
    LB_STAGE("down_gemm", 1, wgemm(3, b->w_d, w.a, d, f, s4, e));
    LB_STAGE("resid_add_len", 1, launch_resid_add(kBF16, w.x1, w.part, s4,
                                                  e.split_stride, y, (long long)B * d, cache_len, B,
                                                  1, s));
  } else {
    const float* X = (const float*)x;
    LB_STAGE("rmsnorm_attn", 1,
             launch_resid_rmsnorm(kF32, x, nullptr, 0, 0, nullptr, b->g1, w.h, B, d, b->eps, s));
    LB_STAGE("qkv_gemm", 1, launch_gemm_f32((const float*)w.h, (const float*)b->w_qkv, w.part, nullptr,
                                            B, b->n_qkv, d, s));
    LB_STAGE("qkv_rope_append", 1,
             launch_qkv_finish(kF32, w.part, 1, 0, B, 1, H, Hkv, dh, cache_len, 0, b->cos_t, b->sin_t,
                               b->max_pos, w.q, k_cache, v_cache, t_max, b->err, s));
    LB_STAGE("attention", 1, launch_attn_f32((const float*)w.q, (const float*)k_cache,
                                             (const float*)v_cache, (float*)w.o, B, 1, 1, H, Hkv, dh,
                                             t_max, cache_len, s));
    LB_STAGE("o_proj_resid_gemm", 1, launch_gemm_f32((const float*)w.o, (const float*)b->w_o,
                                                     (float*)w.x1, X, B, d, H * dh, s));
    LB_STAGE("rmsnorm_mlp", 1,
             launch_resid_rmsnorm(kF32, w.x1, nullptr, 0, 0, nullptr, b->g2, w.h, B, d, b->eps, s));
    LB_STAGE("gate_up_gemm", 1, launch_gemm_f32((const float*)w.h, (const float*)b->w_gu, w.part,
                                                nullptr, B, b->n_gu, d, s));
    LB_STAGE("silu_mul", 1, launch_silu_mul(kF32, w.part, 1, 0, B, f, b->n_gu, 0, w.a, s));
    LB_STAGE("down_resid_gemm", 1, launch_gemm_f32((const float*)w.a, (const float*)b->w_d, (float*)y,
                                                   (const float*)w.x1, B, d, f, s));
    LB_STAGE("increment_lengths", 1,
             launch_resid_add(kF32, nullptr, nullptr, 0, 0, nullptr, 0, cache_len, B, 1, s));
  }
  for (int i = 0; i < B; ++i) b->lens[i] += 1;
  return LB_OK;
}

// ---------------------------------------------------------------- tensor parallelism
// "深入解析Llama MLP模块" page §6.3: with the block split over ranks (Q/K/V and gate/up
// split by output rows, o_proj and down by input columns), each rank computes a partial
// sum of the attention branch and of the MLP branch, and an all-reduce over ranks
// completes each. A shard handle is an ordinary handle created with the rank's head
// counts and intermediate size and given the rank's weight slices; these calls run its
// partial branches. bf16 handles only.
static lb_status tp_check(llama_block* b, const char* who) {
  if (!b) return fail(LB_ERR_INVALID_ARG, "%s: NULL handle", who);
  if (b->dtype != kBF16) return fail(LB_ERR_UNSUPPORTED, "%s: tensor-parallel shards need LB_BF16", who);
  if (!b->has_weights) return fail(LB_ERR_NO_WEIGHTS, "%s: set_weights first", who);
  return LB_OK;
}

lb_status llama_block_tp_attn_prefill(llama_block* b, const void* x, void* o_part, int B, int T,
                                      void* k_cache, void* v_cache, int t_max, int32_t* cache_len,
                                      void* stream) {
  lb_status st = check_cache_args(b, x, o_part, B, k_cache, v_cache, t_max, cache_len, "tp_attn_prefill");
  if (st != LB_OK) return st;
  if ((st = tp_check(b, "tp_attn_prefill")) != LB_OK) return st;
  LB_ON_DEVICE(b, "tp_attn_prefill");
  if (T <= 0) return fail(LB_ERR_INVALID_ARG, "tp_attn_prefill: T must be positive");
  if (T > t_max || T > b->max_pos)
    return fail(LB_ERR_CACHE_FULL, "tp_attn_prefill: T=%d exceeds t_max=%d or max_pos=%d", T, t_max,
                b->max_pos);
  cudaStream_t s = (cudaStream_t)stream;
  const int M = B * T;
  size_t need = 0;
  carve_prefill(b, nullptr, M, &need);
  if ((st = ensure_ws(b, need)) != LB_OK) return st;
  PrefillWs w = carve_prefill(b, b->ws, M, &need);
  const int d = b->d, H = b->H, Hkv = b->Hkv, dh = b->dh;
  b->stage_names.clear();
  if (rope_rows_stale(b, T)) LB_STAGE("rope_table", 1, update_rope_rows(b, 0, T, T, s));
  LB_STAGE("row_stats_attn", 1, launch_row_ssq(x, w.ss1, w.ss2, M, d, cache_len, B, T, b->err, s));
  GemmEpi e1;
  e1.kind = kEpiQkvRope;
  e1.T = T; e1.H = H; e1.Hkv = Hkv; e1.dh = dh; e1.t_max = t_max; e1.max_pos = b->max_pos;
  e1.q_out = w.q; e1.k_cache = k_cache; e1.v_cache = v_cache; e1.pos0 = 0;
  e1.cos_t = b->cos_t; e1.sin_t = b->sin_t; e1.err = b->err;
  e1.row_ss = w.ss1; e1.row_inv_d = 1.f / d; e1.row_eps = b->eps;
  e1.operands_ready = true;  // x and W_qkv: only the epilogue needs row_ssq's statistics
  LB_STAGE("qkv_rope_gemm", 1, launch_gemm_tc(x, b->w_qkv, M, b->n_qkv, d, 256, 1, e1, b->num_sms, s));
  LB_STAGE("attention", 1, launch_attn_tc(w.q, k_cache, v_cache, w.o, B, T, T, H, Hkv, dh, t_max, b->err, s));
  GemmEpi e2;  // this shard's o_proj columns: a partial sum, no residual
  e2.kind = kEpiStore; e2.out = o_part; e2.ldo = d; e2.err = b->err;
  LB_STAGE("o_proj_partial_gemm", 1, launch_gemm_tc(w.o, b->w_o, M, d, H * dh, 256, 1, e2, b->num_sms, s));
  b->lens.assign(B, T);
  return LB_OK;
}

lb_status llama_block_tp_attn_decode(llama_block* b, const void* x, void* o_part, int B, void* k_cache,
                                     void* v_cache, int t_max, int32_t* cache_len, void* stream) {
  lb_status st = check_cache_args(b, x, o_part, B, k_cache, v_cache, t_max, cache_len, "tp_attn_decode");
  if (st != LB_OK) return st;
  if ((st = tp_check(b, "tp_attn_decode")) != LB_OK) return st;
  LB_ON_DEVICE(b, "tp_attn_decode");
  if ((int)b->lens.size() != B)
    return fail(LB_ERR_INVALID_ARG, "tp_attn_decode: the handle knows %d sequence lengths, B=%d",
                (int)b->lens.size(), B);
  for (int i = 0; i < B; ++i)
    if (b->lens[i] < 0 || b->lens[i] + 1 > t_max || b->lens[i] >= b->max_pos)
      return fail(LB_ERR_CACHE_FULL, "tp_attn_decode: sequence %d at length %d cannot grow", i, b->lens[i]);
  cudaStream_t s = (cudaStream_t)stream;
  size_t need = 0;
  carve_decode(b, nullptr, B, t_max, &need);
  if ((st = ensure_ws(b, need)) != LB_OK) return st;
  DecodeWs w = carve_decode(b, b->ws, B, t_max, &need);
  const int d = b->d, H = b->H, Hkv = b->Hkv, dh = b->dh;
  const DecodePlan plan = decode_plan(b, B, b->decode_int8);
  auto wgemm = [&](int i, const void* wbf, const void* act, int Mw, int Kw, int split,
                   const GemmEpi& ep) -> cudaError_t {
    if (plan.w8) return launch_gemm_w8(b->q8[i], b->s8[i], act, Mw, B, Kw, split, ep, b->num_sms, s);
    return launch_gemm_tc(wbf, act, Mw, B, Kw, plan.bn, split, ep, b->num_sms, s);
  };
  b->stage_names.clear();
  {  // dynamic NTK: the rows at the sequences' positions, for this step's base
    int lo = b->lens[0], hi = b->lens[0] + 1;
    for (int v : b->lens) {
      lo = std::min(lo, v);
      hi = std::max(hi, v + 1);
    }
    if (rope_rows_stale(b, hi)) LB_STAGE("rope_table", 1, update_rope_rows(b, lo, hi, hi, s));
  }
  LB_STAGE("rmsnorm_attn", 1,
           launch_resid_rmsnorm(kBF16, x, nullptr, 0, 0, nullptr, nullptr, w.h, B, d, b->eps, s));
  GemmEpi e;
  e.kind = kEpiPartialT; e.out = w.part; e.err = b->err;
  e.ldo = b->n_qkv; e.split_stride = (long long)B * b->n_qkv;
  LB_STAGE("qkv_gemm", 1, wgemm(0, b->w_qkv, w.h, b->n_qkv, d, plan.split[0], e));
  LB_STAGE("qkv_rope_append", 1,
           launch_qkv_finish(kBF16, w.part, plan.split[0], e.split_stride, B, 1, H, Hkv, dh, cache_len, 0,
                             b->cos_t, b->sin_t, b->max_pos, w.q, k_cache, v_cache, t_max, b->err, s));
  LB_STAGE("attention", 2, launch_attn_decode(w.q, k_cache, v_cache, w.o, w.attn_part, B, H, Hkv, dh, t_max,
                                              cache_len, b->err, s));
  e.ldo = d; e.split_stride = (long long)B * d;
  LB_STAGE("o_proj_gemm", 1, wgemm(1, b->w_o, w.o, d, H * dh, plan.split[1], e));
  // the partial sum of this shard's o_proj columns; cache_len += 1
  LB_STAGE("o_partial_len", 1, launch_resid_add(kBF16, nullptr, w.part, plan.split[1], e.split_stride,
                                                o_part, (long long)B * d, cache_len, B, 1, s));
  for (int i = 0; i < B; ++i) b->lens[i] += 1;
  return LB_OK;
}

lb_status llama_block_tp_mlp(llama_block* b, const void* x, const void* o_sum, void* x1, void* m_part,
                             int M, void* stream) {
  lb_status st = tp_check(b, "tp_mlp");
  if (st != LB_OK) return st;
  if (!x || !o_sum || !x1 || !m_part) return fail(LB_ERR_INVALID_ARG, "tp_mlp: NULL argument");
  if (M < 0) return fail(LB_ERR_INVALID_ARG, "tp_mlp: negative row count");
  if (x1 == x || x1 == o_sum || m_part == x1)
    return fail(LB_ERR_INVALID_ARG, "tp_mlp: x1 and m_part must not alias the inputs");
  if (M == 0) return LB_OK;
  LB_ON_DEVICE(b, "tp_mlp");
  cudaStream_t s = (cudaStream_t)stream;
  const int d = b->d, f = b->f;
  b->stage_names.clear();
  size_t need = 0;
  if (M <= 256) {  // decode-sized: swap-AB split-K GEMMs
    carve_decode(b, nullptr, M, 1, &need);
    if ((st = ensure_ws(b, need)) != LB_OK) return st;
    DecodeWs w = carve_decode(b, b->ws, M, 1, &need);
    const DecodePlan plan = decode_plan(b, M, b->decode_int8);
    auto wgemm = [&](int i, const void* wbf, const void* act, int Mw, int Kw, int split,
                     const GemmEpi& ep) -> cudaError_t {
      if (plan.w8) return launch_gemm_w8(b->q8[i], b->s8[i], act, Mw, M, Kw, split, ep, b->num_sms, s);
      return launch_gemm_tc(wbf, act, Mw, M, Kw, plan.bn, split, ep, b->num_sms, s);
    };
    LB_STAGE("resid_add_attn", 1, launch_add_rows(kBF16, x, o_sum, x1, nullptr, M, d, s));
    LB_STAGE("rmsnorm_mlp", 1,
             launch_resid_rmsnorm(kBF16, x1, nullptr, 0, 0, nullptr, nullptr, w.h, M, d, b->eps, s));
    GemmEpi e;
    e.kind = kEpiPartialT; e.out = w.part; e.err = b->err;
    e.ldo = b->n_gu; e.split_stride = (long long)M * b->n_gu;
    LB_STAGE("gate_up_gemm", 1, wgemm(2, b->w_gu, w.h, b->n_gu, d, plan.split[2], e));
    LB_STAGE("silu_mul", 1, launch_silu_mul(kBF16, w.part, plan.split[2], e.split_stride, M, f, b->n_gu, 128,
                                            w.a, s));
    e.ldo = d; e.split_stride = (long long)M * d;
    LB_STAGE("down_gemm", 1, wgemm(3, b->w_d, w.a, d, f, plan.split[3], e));
    LB_STAGE("m_partial", 1, launch_resid_add(kBF16, nullptr, w.part, plan.split[3], e.split_stride, m_part,
                                              (long long)M * d, nullptr, 0, 0, s));
    return LB_OK;
  }
  carve_prefill(b, nullptr, M, &need);
  if ((st = ensure_ws(b, need)) != LB_OK) return st;
  PrefillWs w = carve_prefill(b, b->ws, M, &need);
  // X' = X + (all-reduced attention partial) with its RMSNorm statistic
  LB_STAGE("resid_add_attn", 1, launch_add_rows(kBF16, x, o_sum, x1, w.ss2, M, d, s));
  GemmEpi e3;
  e3.kind = kEpiSwiGLU; e3.out = w.a; e3.ldo = f; e3.f = f; e3.err = b->err;
  e3.row_ss = w.ss2; e3.row_inv_d = 1.f / d; e3.row_eps = b->eps;
  LB_STAGE("gate_up_swiglu_gemm", 1, launch_gemm_tc(x1, b->w_gu, M, b->n_gu, d, 256, 1, e3, b->num_sms, s));
  GemmEpi e4;  // this shard's down columns: a partial sum, no residual
  e4.kind = kEpiStore; e4.out = m_part; e4.ldo = d; e4.err = b->err;
  LB_STAGE("down_partial_gemm", 1, launch_gemm_tc(w.a, b->w_d, M, d, f, 256, 1, e4, b->num_sms, s));
  return LB_OK;
}

lb_status llama_block_tp_add(const void* a, const void* b_in, void* out, int rows, int d, lb_dtype dtype,
                             void* stream) {
  if (rows < 0 || d <= 0 || d % 8) return fail(LB_ERR_INVALID_ARG, "tp_add: bad shape (d %% 8 == 0)");
  if (rows == 0) return LB_OK;
  if (!a || !b_in || !out) return fail(LB_ERR_INVALID_ARG, "tp_add: NULL argument");
  const int dt = dtype == LB_F32 ? kF32 : kBF16;
  LB_CUDA(launch_add_rows(dt, a, b_in, out, nullptr, rows, d, (cudaStream_t)stream));
  return LB_OK;
}

lb_status llama_block_enable_timing(llama_block* b, int enable) {
  if (!b) return fail(LB_ERR_INVALID_ARG, "enable_timing: NULL handle");
  LB_ON_DEVICE(b, "enable_timing");
  if (enable && b->ev.empty()) {
    b->ev.resize(2 * kMaxStages);
    for (auto& e : b->ev) LB_CUDA(cudaEventCreate(&e));
  }
  b->timing = enable != 0;
  return LB_OK;
}

lb_status llama_block_stage_times(llama_block* b, float* ms, int max_stages, int* n_stages) {
  if (!b || !n_stages) return fail(LB_ERR_INVALID_ARG, "stage_times: NULL argument");
  if (!b->timing) return fail(LB_ERR_INVALID_ARG, "stage_times: timing is not enabled");
  LB_ON_DEVICE(b, "stage_times");
  const int n = std::min((int)b->stage_names.size(), kMaxStages);
  *n_stages = n;
  for (int i = 0; i < n && i < max_stages && ms; ++i) {
    LB_CUDA(cudaEventSynchronize(b->ev[2 * i + 1]));
    LB_CUDA(cudaEventElapsedTime(&ms[i], b->ev[2 * i], b->ev[2 * i + 1]));
  }
  return LB_OK;
}

const char* llama_block_stage_name(const llama_block* b, int i) {
  if (!b || i < 0 || i >= (int)b->stage_names.size()) return "";
  return b->stage_names[i];
}

unsigned long long llama_block_launch_count(const llama_block* b) { return b ? b->launches : 0; }

static const char* describe_err(int code) {
  if (code >= kErrWaitBase && code < kErrWaitBase + 0x100) return "a bounded device wait ran out";
  return "a device-side bounds guard fired (cache index or RoPE position out of range)";
}

// Read a device error word and clear it when it is set.
static cudaError_t take_err_word(int* word, int* code) {
  *code = 0;
  if (!word) return cudaSuccess;
  cudaError_t e = cudaMemcpy(code, word, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && *code != 0) e = cudaMemset(word, 0, sizeof(int));
  return e;
}

static cudaError_t noalloc_take_error(int* code);  // decode_attn_static_scratch's word

lb_status llama_block_sync_status(llama_block* b, void* stream) {
  DeviceGuard dg(b ? b->device : -1);
  if (b && !dg.ok) return fail(LB_ERR_CUDA, "sync_status: cannot select the handle's device");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return fail(LB_ERR_CUDA, "sync_status: %s", cudaGetErrorString(e));
  int code = 0;
  if (b) {
    LB_CUDA(take_err_word(b->err, &code));
  } else {
    // the standalone entry points of the current device: the word they share (looked up,
    // never created here, so this allocates nothing) and the allocation-free decode
    // attention's own word; both are cleared, the first code set is reported
    int c_noalloc = 0;
    LB_CUDA(take_err_word(existing_standalone_err_word(), &code));
    LB_CUDA(noalloc_take_error(&c_noalloc));
    if (code == 0) code = c_noalloc;
  }
  if (code == 0) return LB_OK;
  const bool wait = code >= kErrWaitBase && code < kErrWaitBase + 0x100;
  return fail(wait ? LB_ERR_TIMEOUT : LB_ERR_CACHE_FULL, "device error 0x%x: %s", code,
              describe_err(code));
}

lb_status llama_block_selftest_timeout(long long budget_ns, void* stream) {
  if (budget_ns <= 0) return fail(LB_ERR_INVALID_ARG, "selftest_timeout: budget must be positive");
  int* word = standalone_err_word();
  if (!word) return fail(LB_ERR_CUDA, "selftest_timeout: no device");
  LB_CUDA(launch_selftest_timeout(word, (unsigned long long)budget_ns, (cudaStream_t)stream));
  return LB_OK;
}

// ------------------------------------------------------------------ standalone
static lb_status check_dtype(lb_dtype dt, const char* who) {
  if (dt != LB_F32 && dt != LB_BF16) return fail(LB_ERR_INVALID_ARG, "%s: bad dtype", who);
  return LB_OK;
}

lb_status rmsnorm(const void* x, const void* g, void* y, int rows, int d, float eps,
                  lb_dtype dtype, void* stream) {
  if (check_dtype(dtype, "rmsnorm") != LB_OK) return LB_ERR_INVALID_ARG;
  if (rows < 0 || d <= 0 || !(eps > 0.f)) return fail(LB_ERR_INVALID_ARG, "rmsnorm: bad size");
  if (rows == 0) return LB_OK;  // nothing to do; empty tensors may carry NULL pointers
  if (!x || !g || !y) return fail(LB_ERR_INVALID_ARG, "rmsnorm: NULL pointer");
  if (d % 8 != 0 || d > 8192)
    return fail(LB_ERR_UNSUPPORTED, "rmsnorm: d must be a multiple of 8 and <= 8192");
  LB_CUDA(launch_resid_rmsnorm(dtype, x, nullptr, 0, 0, nullptr, g, y, rows, d, eps,
                               (cudaStream_t)stream));
  return LB_OK;
}

lb_status rope_apply(void* x, const int32_t* pos, int B, int T, int n_heads, int head_dim,
                     float base, lb_dtype dtype, void* stream) {
  if (check_dtype(dtype, "rope_apply") != LB_OK) return LB_ERR_INVALID_ARG;
  if (!x || !pos) return fail(LB_ERR_INVALID_ARG, "rope_apply: NULL pointer");
  if (B < 0 || T < 0 || n_heads <= 0 || head_dim <= 0 || head_dim % 2 || !(base > 0.f))
    return fail(LB_ERR_INVALID_ARG, "rope_apply: bad size");
  LB_CUDA(launch_rope_apply(dtype, x, pos, B, T, n_heads, head_dim, (double)base,
                            (cudaStream_t)stream));
  return LB_OK;
}

lb_status causal_attn(const void* q, const void* k, const void* v, void* o, int B, int Tq, int Tk,
                      int n_heads, int n_kv_heads, int head_dim, int k_stride_T, lb_dtype dtype,
                      void* stream) {
  if (check_dtype(dtype, "causal_attn") != LB_OK) return LB_ERR_INVALID_ARG;
  if (!q || !k || !v || !o) return fail(LB_ERR_INVALID_ARG, "causal_attn: NULL pointer");
  if (B < 0 || Tq < 1 || Tk < Tq || k_stride_T < Tk || n_heads <= 0 || n_kv_heads <= 0)
    return fail(LB_ERR_INVALID_ARG, "causal_attn: need 1 <= Tq <= Tk <= k_stride_T");
  if (head_dim != 64 && head_dim != 128)
    return fail(LB_ERR_UNSUPPORTED, "causal_attn: head_dim %d not in {64,128}", head_dim);
  if (n_heads % n_kv_heads) return fail(LB_ERR_UNSUPPORTED, "causal_attn: n_heads %% n_kv_heads");
  if (dtype == LB_BF16 && (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)o) & 15))
    return fail(LB_ERR_INVALID_ARG, "causal_attn: bf16 q, k, v and o must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == LB_BF16) {
    int* err = standalone_err_word();
    LB_CUDA(launch_attn_tc(q, k, v, o, B, Tq, Tk, n_heads, n_kv_heads, head_dim, k_stride_T, err, s));
  } else {
    LB_CUDA(launch_attn_f32((const float*)q, (const float*)k, (const float*)v, (float*)o, B, Tq, Tk,
                            n_heads, n_kv_heads, head_dim, k_stride_T, nullptr, s));
  }
  return LB_OK;
}

lb_status swiglu_mlp(const void* h, const void* w_gate, const void* w_up, const void* w_down,
                     void* y, int M, int d, int f, lb_dtype dtype, void* stream) {
  if (check_dtype(dtype, "swiglu_mlp") != LB_OK) return LB_ERR_INVALID_ARG;
  if (!h || !w_gate || !w_up || !w_down || !y) return fail(LB_ERR_INVALID_ARG, "swiglu_mlp: NULL pointer");
  if (M < 0 || d <= 0 || f <= 0) return fail(LB_ERR_INVALID_ARG, "swiglu_mlp: bad size");
  if (dtype == LB_BF16 && (d % 64 || f % 8))
    return fail(LB_ERR_UNSUPPORTED, "swiglu_mlp: bf16 needs d %% 64 == 0 and f %% 8 == 0");
  if (M == 0) return LB_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t es = dtype == LB_F32 ? 4 : 2;
  const int f_pad = dtype == LB_BF16 ? (f + 127) / 128 * 128 : f;
  const int n_gu = 2 * f_pad;
  char* tmp = nullptr;
  const size_t wbytes = align_up((size_t)n_gu * d * es, 256);
  const size_t abytes = align_up((size_t)M * f_pad * es, 256);
  const size_t gbytes = dtype == LB_F32 ? (size_t)M * n_gu * 4 : 0;
  LB_CUDA(cudaMallocAsync((void**)&tmp, wbytes + abytes + gbytes, s));
  lb_status st = LB_OK;
  auto run = [&]() -> lb_status {
    LB_CUDA(cudaMemsetAsync(tmp, 0, wbytes, s));
    if (dtype == LB_F32) {
      LB_CUDA(cudaMemcpyAsync(tmp, w_gate, (size_t)f * d * es, cudaMemcpyDeviceToDevice, s));
      LB_CUDA(cudaMemcpyAsync(tmp + (size_t)f * d * es, w_up, (size_t)f * d * es,
                              cudaMemcpyDeviceToDevice, s));
      float* gu = (float*)(tmp + wbytes + abytes);
      LB_CUDA(launch_gemm_f32((const float*)h, (const float*)tmp, gu, nullptr, M, n_gu, d, s));
      LB_CUDA(launch_silu_mul(kF32, gu, 1, 0, M, f, n_gu, 0, tmp + wbytes, s));
      LB_CUDA(launch_gemm_f32((const float*)(tmp + wbytes), (const float*)w_down, (float*)y,
                              nullptr, M, d, f, s));
    } else {
      const size_t blk = 128 * (size_t)d * es;
      const int full = f / 128, rem = f - full * 128;
      if (full > 0) {
        LB_CUDA(cudaMemcpy2DAsync(tmp, 2 * blk, w_gate, blk, blk, full, cudaMemcpyDeviceToDevice, s));
        LB_CUDA(cudaMemcpy2DAsync(tmp + blk, 2 * blk, w_up, blk, blk, full,
                                  cudaMemcpyDeviceToDevice, s));
      }
      if (rem > 0) {
        const size_t src = (size_t)full * blk;
        LB_CUDA(cudaMemcpyAsync(tmp + 2 * src, (const char*)w_gate + src, rem * d * es,
                                cudaMemcpyDeviceToDevice, s));
        LB_CUDA(cudaMemcpyAsync(tmp + 2 * src + blk, (const char*)w_up + src, rem * d * es,
                                cudaMemcpyDeviceToDevice, s));
      }
      const int nsm = num_sms_of_current_device();
      GemmEpi e3;
      e3.kind = kEpiSwiGLU; e3.out = tmp + wbytes; e3.ldo = f; e3.f = f;
      e3.err = standalone_err_word();
      LB_CUDA(launch_gemm_tc(h, tmp, M, n_gu, d, 256, 1, e3, nsm, s));
      GemmEpi e4;
      e4.kind = kEpiStore; e4.out = y; e4.ldo = d; e4.err = e3.err;
      LB_CUDA(launch_gemm_tc(tmp + wbytes, w_down, M, d, f, 256, 1, e4, nsm, s));
    }
    return LB_OK;
  };
  st = run();
  cudaFreeAsync(tmp, s);
  return st;
}

}  // extern "C"

// ------------------------------------------------------------------ stack of blocks
// L decoder layers applied in sequence (the "x L blocks" of the mechanics page's
// chapter-02 diagram; LMDrive page §1, 32 LlamaDecoderLayers). Each layer is a
// llama_block with its own weights and its own caller-owned KV cache; the stack
// owns two ping-pong activation buffers and one device length array per layer.
struct llama_stack {
  std::vector<llama_block*> layers;
  int device = 0;  // the device of every layer (current at creation)
  int d = 0;
  size_t esz = 0;
  void* act[2] = {nullptr, nullptr};
  size_t act_bytes = 0;
  int32_t* lens = nullptr;  // [layers][B]
  int lens_cap = 0;
};

extern "C" {

void llama_stack_destroy(llama_stack* st) {
  if (!st) return;
  DeviceGuard dg(st->device);
  cudaDeviceSynchronize();
  for (llama_block* b : st->layers) llama_block_destroy(b);
  for (void* p : {st->act[0], st->act[1], (void*)st->lens})
    if (p) cudaFree(p);
  delete st;
}

lb_status llama_stack_create(int n_layers, int d, int n_heads, int n_kv_heads, int head_dim, int f,
                             float eps, float rope_base, lb_dtype dtype, int max_pos,
                             llama_stack** out) {
  if (!out) return fail(LB_ERR_INVALID_ARG, "stack_create: out is NULL");
  *out = nullptr;
  if (n_layers <= 0) return fail(LB_ERR_INVALID_ARG, "stack_create: n_layers must be positive");
  llama_stack* st = new llama_stack();
  if (cudaGetDevice(&st->device) != cudaSuccess) {
    delete st;
    return fail(LB_ERR_CUDA, "stack_create: no CUDA device");
  }
  for (int l = 0; l < n_layers; ++l) {
    llama_block* b = nullptr;
    const lb_status r =
        llama_block_create(d, n_heads, n_kv_heads, head_dim, f, eps, rope_base, dtype, max_pos, &b);
    if (r != LB_OK) {
      const std::string msg = g_last_error;
      llama_stack_destroy(st);
      return fail(r, "stack_create: layer %d: %s", l, msg.c_str());
    }
    st->layers.push_back(b);
  }
  st->d = d;
  st->esz = dtype == LB_F32 ? 4 : 2;
  *out = st;
  return LB_OK;
}

llama_block* llama_stack_layer(llama_stack* st, int layer) {
  if (!st || layer < 0 || layer >= (int)st->layers.size()) return nullptr;
  return st->layers[layer];
}

lb_status llama_stack_set_lengths(llama_stack* st, const int32_t* lens_host, int B) {
  if (!st) return fail(LB_ERR_INVALID_ARG, "stack_set_lengths: NULL stack");
  for (llama_block* b : st->layers) {
    const lb_status r = llama_block_set_lengths(b, lens_host, B);
    if (r != LB_OK) return r;
  }
  return LB_OK;
}

}  // extern "C"

enum StackOp { kStackPrefill, kStackExtend, kStackDecode };

static lb_status stack_run(llama_stack* st, StackOp op, const void* x, void* y, int B, int T,
                           void* const* k_caches, void* const* v_caches, int t_max,
                           int32_t* cache_len, void* stream) {
  const char* who = op == kStackPrefill ? "stack_prefill" : op == kStackExtend ? "stack_extend" : "stack_decode";
  if (!st || !x || !y || !k_caches || !v_caches || !cache_len)
    return fail(LB_ERR_INVALID_ARG, "%s: NULL argument", who);
  if (B <= 0 || T <= 0) return fail(LB_ERR_INVALID_ARG, "%s: B and T must be positive", who);
  if (x == y) return fail(LB_ERR_INVALID_ARG, "%s: y must not alias x", who);
  LB_ON_DEVICE(st, who);
  const int n = (int)st->layers.size();
  for (int l = 0; l < n; ++l)
    if (!k_caches[l] || !v_caches[l])
      return fail(LB_ERR_INVALID_ARG, "%s: NULL cache pointer for layer %d", who, l);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t act = (size_t)B * T * st->d * st->esz;
  if (n > 1 && act > st->act_bytes) {
    LB_CUDA(cudaDeviceSynchronize());
    for (int i = 0; i < 2; ++i) {
      if (st->act[i]) LB_CUDA(cudaFree(st->act[i]));
      st->act[i] = nullptr;
    }
    st->act_bytes = 0;
    LB_CUDA(cudaMalloc(&st->act[0], act));
    LB_CUDA(cudaMalloc(&st->act[1], act));
    st->act_bytes = act;
  }
  if (n * B > st->lens_cap) {
    LB_CUDA(cudaDeviceSynchronize());
    if (st->lens) LB_CUDA(cudaFree(st->lens));
    st->lens = nullptr;
    st->lens_cap = 0;
    LB_CUDA(cudaMalloc(&st->lens, (size_t)n * B * sizeof(int32_t)));
    st->lens_cap = n * B;
  }
  // every layer starts from the caller's lengths and updates its own copy
  for (int l = 0; l < n; ++l)
    LB_CUDA(cudaMemcpyAsync(st->lens + (size_t)l * B, cache_len, B * sizeof(int32_t),
                            cudaMemcpyDeviceToDevice, s));
  const void* in = x;
  for (int l = 0; l < n; ++l) {
    void* out = l == n - 1 ? y : st->act[l & 1];
    int32_t* ll = st->lens + (size_t)l * B;
    lb_status r;
    if (op == kStackPrefill)
      r = llama_block_prefill(st->layers[l], in, out, B, T, k_caches[l], v_caches[l], t_max, ll, stream);
    else if (op == kStackExtend)
      r = llama_block_extend(st->layers[l], in, out, B, T, k_caches[l], v_caches[l], t_max, ll, stream);
    else
      r = llama_block_decode(st->layers[l], in, out, B, k_caches[l], v_caches[l], t_max, ll, stream);
    if (r != LB_OK) {
      const std::string msg = g_last_error;
      return fail(r, "%s: layer %d: %s", who, l, msg.c_str());
    }
    in = out;
  }
  LB_CUDA(cudaMemcpyAsync(cache_len, st->lens + (size_t)(n - 1) * B, B * sizeof(int32_t),
                          cudaMemcpyDeviceToDevice, s));
  return LB_OK;
}

extern "C" {

lb_status llama_stack_prefill(llama_stack* st, const void* x, void* y, int B, int T,
                              void* const* k_caches, void* const* v_caches, int t_max,
                              int32_t* cache_len, void* stream) {
  return stack_run(st, kStackPrefill, x, y, B, T, k_caches, v_caches, t_max, cache_len, stream);
}

lb_status llama_stack_extend(llama_stack* st, const void* x, void* y, int B, int T,
                             void* const* k_caches, void* const* v_caches, int t_max,
                             int32_t* cache_len, void* stream) {
  return stack_run(st, kStackExtend, x, y, B, T, k_caches, v_caches, t_max, cache_len, stream);
}

lb_status llama_stack_decode(llama_stack* st, const void* x, void* y, int B, void* const* k_caches,
                             void* const* v_caches, int t_max, int32_t* cache_len, void* stream) {
  return stack_run(st, kStackDecode, x, y, B, 1, k_caches, v_caches, t_max, cache_len, stream);
}

}  // extern "C"

// ------------------------------------------------------------------ static-scratch decode attention
// For callers that may not allocate device memory, decode attention with its
// split-KV partials kept in a fixed array of this file instead of a caller- or
// library-allocated workspace. The array (kNoAllocScratchFloats floats, 24 MiB)
// is part of the library image: every GPU that loads the library holds it until
// the process exits. Its device address is looked up once per device.
static constexpr size_t kNoAllocScratchFloats = (size_t)6 << 20;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];
static __device__ int g_noalloc_err;

struct NoAllocSlot {
  float* scratch = nullptr;
  int* err = nullptr;
};
static std::mutex g_noalloc_mu;
static std::map<int, NoAllocSlot> g_noalloc_slots;

// Read and clear the current device's word (nothing to read before the first call there).
static cudaError_t noalloc_take_error(int* code) {
  *code = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int* word = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    auto it = g_noalloc_slots.find(dev);
    if (it != g_noalloc_slots.end()) word = it->second.err;
  }
  return take_err_word(word, code);
}

extern "C" lb_status decode_attn_static_scratch(const void* q, const void* k, const void* v,
                                                void* o, const int32_t* kv_len, int B,
                                                int n_heads, int n_kv_heads, int head_dim,
                                                int k_stride_T, void* stream) {
  if (!q || !k || !v || !o || !kv_len)
    return fail(LB_ERR_INVALID_ARG, "decode_attn_static_scratch: NULL pointer");
  if (B <= 0 || n_heads <= 0 || n_kv_heads <= 0 || k_stride_T <= 0)
    return fail(LB_ERR_INVALID_ARG, "decode_attn_static_scratch: sizes must be positive");
  if (head_dim != 64 && head_dim != 128)
    return fail(LB_ERR_UNSUPPORTED, "decode_attn_static_scratch: head_dim %d not in {64,128}", head_dim);
  if (n_heads % n_kv_heads)
    return fail(LB_ERR_UNSUPPORTED, "decode_attn_static_scratch: n_heads %% n_kv_heads != 0");
  if (((uintptr_t)k | (uintptr_t)v) & 15)
    return fail(LB_ERR_INVALID_ARG, "decode_attn_static_scratch: k and v must be 16-byte aligned");
  const size_t need = (size_t)B * n_heads * decode_attn_chunks(k_stride_T) * (head_dim + 2);
  if (need > kNoAllocScratchFloats)
    return fail(LB_ERR_INVALID_ARG,
                "decode_attn_static_scratch: B*n_heads*ceil(k_stride_T/512)*(head_dim+2) = %zu "
                "floats exceeds the fixed scratch of %zu floats",
                need, kNoAllocScratchFloats);
  int dev = 0;
  LB_CUDA(cudaGetDevice(&dev));
  NoAllocSlot slot;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    auto it = g_noalloc_slots.find(dev);
    if (it == g_noalloc_slots.end()) {
      // first call on this device: resolve the device addresses of the arrays
      LB_CUDA(cudaGetSymbolAddress((void**)&slot.scratch, g_noalloc_scratch));
      LB_CUDA(cudaGetSymbolAddress((void**)&slot.err, g_noalloc_err));
      g_noalloc_slots[dev] = slot;
    } else {
      slot = it->second;
    }
  }
  // The partials need no clearing: every (sequence, head, chunk) slot the combine
  // step reads is written by this call's split kernel first.
  LB_CUDA(launch_attn_decode(q, k, v, o, slot.scratch, B, n_heads, n_kv_heads, head_dim, k_stride_T,
                             kv_len, slot.err, (cudaStream_t)stream));
  return LB_OK;
}
