// attn_tc.cu — causal softmax attention for prefill on the tcgen05 tensor cores
// (LMDrive page §2.3 LlamaAttention; "LLM 核心机制交互讲义" §02.1 causal mask):
//
//   O = softmax(Q K^T / sqrt(d_h) + M) V,   M_ij = 0 for key j <= query position i,
//                                            -inf otherwise,
// with GQA: query head h reads KV head h / (H / H_kv) (repeat_kv without
// materialising the repeat).
//
// Work unit: one 128-row query tile of one (sequence, head); it needs one 128-key
// step per K/V tile up to its diagonal. The kernel is persistent: one CTA per SM walks
// its units in a snake order over the list sorted heaviest first (round r takes units
// r*G .. r*G + G - 1, forwards on even rounds and backwards on odd ones), and every
// pipeline below runs across unit boundaries, so the next unit's Q load and first
// score tiles overlap the current unit's last steps and its output write.
//   warp 0       TMA producer: the Q of units 0 and 1, then K one ring ahead of V (K_0,
//                K_1, K_2, then V_g, K_{g+3} per step g). A K (V) stage is reused once
//                the S (PV) product that read it completed. It never waits for a Q
//                buffer: the epilogue loads the later units' Q (below).
//   warp 10      issues S(g) = Q K^T into TMEM score buffer g % 3, so S(g+1) and
//                S(g+2) are computed while the softmax works on S(g); S(g) overwrites
//                P(g-3) and therefore waits for PV(g-3) to complete.
//   warp 1       TMEM allocation; issues O += P(g) V, reading P(g) (bf16, written by
//                the softmax over its own buffer's score columns) straight from TMEM
//                with V MN-major in shared memory. One wait covers both inputs: the
//                softmax warps and the V load arrive on the same barrier. The first PV
//                of a unit waits until the previous unit's O has been read out.
//                Two issuing threads because a tcgen05.mma issue blocks until the
//                tensor pipe takes it: one thread's barrier waits and bookkeeping
//                between its MMAs would leave the pipe idle, the other's MMAs fill
//                those gaps.
//   warps 2..9   softmax, two warps per TMEM lane quarter: warps 2..5 take score
//                columns (keys) 0..63 of each row, warps 6..9 keys 64..127. The two
//                halves of a row swap their partial maxima through shared memory (a
//                64-thread named barrier per lane quarter) and share one reference
//                max, so their partial row sums and their halves of P belong to the
//                same O. Online max/sum in fp32 with log2(e)/sqrt(d_h) folded into the
//                exponent's FMA; the reference max only moves (and O is rescaled in
//                TMEM, each half rescaling half of O's columns) when a row's max grows
//                by more than 2^8, so most steps skip the rescale; P <= 2^8 stays exact
//                enough in bf16 and the final O / l uses the same reference.
//                At the end of a unit they hand their half-row sums to the epilogue
//                warps (a two-slot ring in shared memory) and go on with the next unit.
//   warps 11..14 epilogue: wait for the unit's last PV, read O out of TMEM (which
//                releases it to the next unit's PVs), normalise, stage the rows in the
//                unit's Q buffer (its last QK^T has completed) and store the tile with
//                TMA. Once the store has read the buffer, the same thread loads the Q
//                of unit k + 2 into it: a producer that waited for the buffer held
//                back the K/V loads behind it and stalled the PVs at unit changes.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace lb {

constexpr int kAttnTcThreads = 480;
constexpr float kRescaleLog2 = 8.0f;

// ---------------------------------------------------------------- softmax arithmetic
// Three-input max (sm_100): one instruction per two new scores.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Barrier for the two softmax warps that share a TMEM lane quarter (ids 1..4;
// id 0 is __syncthreads). Both warps execute exactly the same sequence of these.
__device__ __forceinline__ void quarter_bar(int quarter) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
}
// tcgen05.mma with shared-memory operand descriptors given as 32-bit (low, high)
// words: the low word holds the start address and the leading byte offset, so a
// K-step only adds a constant to it (addresses stay below 2^18 bytes, so the
// address field never carries into the next one).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "mov.b64 a, {%1, %5};\n\t"
      "mov.b64 b, {%2, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, {%6, %6, %6, %6}, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(hi), "r"(0u));
}
// Same with the A operand in TMEM.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 b;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "mov.b64 b, {%2, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b, %3, {%6, %6, %6, %6}, p;\n\t}" ::"r"(
          d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(hi), "r"(0u));
}

// Barrier for the 128 epilogue threads (id 5).
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 5, 128;" ::: "memory"); }

template <int DH>
struct AttnCfg {
  static constexpr int BQ = 128, BKV = 128;
  static constexpr int NS = 3;                   // score buffers in TMEM
  static constexpr int KST = 2, VST = 2;         // K and V ring stages
  static constexpr int PANELS = DH / 64;         // 64-column, 128-byte swizzled panels
  static constexpr int PANEL_BYTES = 128 * 128;  // one panel of a 128-row tile
  static constexpr int Q_BYTES = BQ * DH * 2;
  static constexpr int KV_BYTES = BKV * DH * 2;
  static constexpr int XCH_FLOATS = 8 * 128;     // row maxima [2 steps][2 halves], row sums [2 units][2 halves]
  static constexpr int SMEM =
      2 * Q_BYTES + (KST + VST) * KV_BYTES + XCH_FLOATS * 4 + 256 + 1024;
  static constexpr int O_COL = NS * 128;         // S buffers at columns 0, 128, 256; O after
  static constexpr int TMEM_COLS = 512;
};

// One work unit: a 128-row query tile of sequence b, query head h (KV head hk);
// n = number of 128-key steps (K/V tiles up to the tile's last row).
struct AttnUnit {
  int b, h, hk, q0, n;
};

__device__ __forceinline__ AttnUnit attn_unit(int U, int B, int Tq, int Tk, int H, int Hkv) {
  const int ntiles = (Tq + 127) / 128;
  const int tile = ntiles - 1 - U / (B * H);  // heaviest tiles first
  const int bh = U % (B * H);
  AttnUnit u;
  u.h = bh % H;
  u.b = bh / H;
  u.hk = u.h / (H / Hkv);
  u.q0 = tile * 128;
  u.n = min(Tk - Tq + u.q0 + 127, Tk - 1) / 128 + 1;  // >= 1: key 0 is visible to every row
  return u;
}

// The k-th unit of CTA c out of G: snake order over the heaviest-first list.
__device__ __forceinline__ int attn_unit_index(int k, int c, int G) {
  return k * G + ((k & 1) ? G - 1 - c : c);
}

// Walks this CTA's (unit, step) sequence; g counts steps over all units.
struct AttnCursor {
  int k, j, g, nunits;
  AttnUnit u;
  int B, Tq, Tk, H, Hkv;
  __device__ __forceinline__ void init(int nu, int B_, int Tq_, int Tk_, int H_, int Hkv_) {
    k = 0, j = 0, g = 0, nunits = nu;
    B = B_, Tq = Tq_, Tk = Tk_, H = H_, Hkv = Hkv_;
    if (nunits > 0) u = attn_unit(attn_unit_index(0, blockIdx.x, gridDim.x), B, Tq, Tk, H, Hkv);
  }
  __device__ __forceinline__ bool valid() const { return k < nunits; }
  __device__ __forceinline__ void advance() {
    ++g;
    if (++j == u.n) {
      j = 0;
      if (++k < nunits) u = attn_unit(attn_unit_index(k, blockIdx.x, gridDim.x), B, Tq, Tk, H, Hkv);
    }
  }
};

template <int DH>
__global__ void __launch_bounds__(kAttnTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   int B, int Tq, int Tk, int H, int Hkv, float scale_log2, int* err) {
  using C = AttnCfg<DH>;
  constexpr int NS = C::NS, KST = C::KST, VST = C::VST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                     // 2 buffers: Q of units k % 2, then their output
  uint8_t* sK = sQ + 2 * C::Q_BYTES;      // KST stages
  uint8_t* sV = sK + KST * C::KV_BYTES;   // VST stages
  float* xch = reinterpret_cast<float*>(sV + VST * C::KV_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(xch + C::XCH_FLOATS);
  uint64_t* q_full = bars;                // [2]
  uint64_t* k_full = q_full + 2;          // [KST]
  // A K stage is free once the S product that read it has completed (s_full), a V
  // stage once its PV product has (o_full): the producer waits on those barriers.
  uint64_t* s_full = k_full + KST;        // [NS] score buffers
  // [NS]: step g's P written (8 softmax warps) and its V tile landed (the producer's
  // arrival with the tile's bytes), so one wait covers both inputs of PV(g)
  uint64_t* pv_ready = s_full + NS;
  uint64_t* o_full = pv_ready + NS;       // [NS]: PV(g) completes a phase of o_full[g % NS]
  uint64_t* o_free = o_full + NS;         // a unit's O has been read out of TMEM
  uint64_t* l_ready = o_free + 1;         // [2]: a unit's row sums handed to the epilogue
  uint64_t* xsum_free = l_ready + 2;      // [2]: ... and read by it
  uint64_t* drain = xsum_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int off = Tk - Tq;  // query row i sits at position off + i
  // units of this CTA: full rounds, plus one in the last partial round if its slot exists
  const int total = ((Tq + 127) / 128) * B * H;
  const int G = gridDim.x, rounds = total / G, rem = total % G;
  const int nunits = rounds + (((rounds & 1) ? G - 1 - (int)blockIdx.x : (int)blockIdx.x) < rem);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) mbar_init(&q_full[i], 1);
    for (int i = 0; i < KST; ++i) mbar_init(&k_full[i], 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&pv_ready[i], 9);  // one arrival per softmax warp + the V load
      mbar_init(&o_full[i], 1);
    }
    mbar_init(o_free, 4);  // one arrival per epilogue warp
    for (int i = 0; i < 2; ++i) {
      mbar_init(&l_ready[i], 8);    // softmax warps
      mbar_init(&xsum_free[i], 4);  // epilogue warps
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  if (warp == 0) {
    if (lane == 0 && nunits > 0) {
      // ---------------- TMA producer
      // Q of units 0 and 1 (both buffers are free); the epilogue's storer loads the Q of
      // unit k + 2 into unit k's buffer once the output staged there has been stored.
      auto load_q = [&](int k, const AttnUnit& u) -> bool {
        const int qb = k & 1;
        mbar_arrive_expect_tx(&q_full[qb], C::Q_BYTES);
        for (int p = 0; p < C::PANELS; ++p)
          tma_load_3d(sQ + qb * C::Q_BYTES + p * C::PANEL_BYTES, &tmQ, &q_full[qb], p * 64, u.q0,
                      u.b * H + u.h);
        return true;
      };
      auto load_kv = [&](bool is_k, const AttnCursor& c) -> bool {
        const int ns = is_k ? KST : VST;
        const int st = c.g % ns;
        uint64_t* full = is_k ? &k_full[st] : &pv_ready[c.g % NS];
        // the stage's previous tile (step g - ns) is free once its product completed
        const int prev = c.g - ns;
        if (prev >= 0 && !mbar_wait(is_k ? &s_full[prev % NS] : &o_full[prev % NS],
                                    (prev / NS) & 1, err, 0x21))
          return false;
        mbar_arrive_expect_tx(full, C::KV_BYTES);
        uint8_t* dst = (is_k ? sK : sV) + st * C::KV_BYTES;
        for (int p = 0; p < C::PANELS; ++p)
          tma_load_3d(dst + p * C::PANEL_BYTES, is_k ? &tmK : &tmV, full, p * 64, c.j * C::BKV,
                      c.u.b * Hkv + c.u.hk);
        return true;
      };
      AttnCursor vc, kc;  // V at step g, K at step g + NS
      vc.init(nunits, B, Tq, Tk, H, Hkv);
      kc.init(nunits, B, Tq, Tk, H, Hkv);
      bool ok = load_q(0, vc.u);
      if (nunits > 1) load_q(1, attn_unit(attn_unit_index(1, blockIdx.x, G), B, Tq, Tk, H, Hkv));
      for (int i = 0; i < NS && ok && kc.valid(); ++i, kc.advance()) ok = load_kv(true, kc);
      int last_g = -1;  // last step whose V was issued
      for (; ok && vc.valid(); vc.advance()) {
        ok = load_kv(false, vc);
        if (!ok) break;
        last_g = vc.g;
        if (kc.valid()) {
          ok = load_kv(true, kc);
          kc.advance();
        }
      }
      pdl_trigger();
      // every issued load must land before the CTA may exit
      for (int i = max(0, last_g - VST + 1); i <= last_g; ++i)
        mbar_wait(&pv_ready[i % NS], (i / NS) & 1, err, 0x22);
      for (int i = max(0, kc.g - KST); i < kc.g; ++i)
        mbar_wait(&k_full[i % KST], (i / KST) & 1, err, 0x22);
      for (int k = max(0, nunits - 2); k < nunits; ++k)
        mbar_wait(&q_full[k & 1], (k >> 1) & 1, err, 0x22);
    }
  } else if (warp == 1 || warp == 10) {
    // ---------------- MMA issue, split over two threads in different warps: warp 10
    // issues the S products, warp 1 the PV products. A tcgen05.mma issue blocks until
    // the tensor pipe takes it, so whatever one issuing thread does between its MMAs
    // (barrier waits, bookkeeping) would leave the pipe idle; with two issuers the
    // other's MMAs fill those gaps. S(g) overwrites P(g - NS), which PV(g - NS) reads:
    // the S thread waits for that PV to complete (o_full) before issuing S(g).
    constexpr uint32_t DHI = (1024u >> 4) | (1u << 14) | (2u << 29);  // SBO 1 KB, sm_100, SW128
    constexpr uint32_t KVD = C::KV_BYTES >> 4, PD = C::PANEL_BYTES >> 4;
    if (warp == 10 && lane == 0 && nunits > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t QD = C::Q_BYTES >> 4;
      const uint32_t q_lo0 = (smem_u32(sQ) >> 4) | (1u << 16);  // LBO 16 B (K-major)
      const uint32_t k_lo0 = (smem_u32(sK) >> 4) | (1u << 16);
      AttnCursor sc;
      sc.init(nunits, B, Tq, Tk, H, Hkv);
      bool ok = true;
      uint32_t s_buf = 0, s_ph = 0, k_st = 0, k_ph = 0;
      for (; ok && sc.valid(); sc.advance()) {
        // the buffer's previous P (step g - NS) has been read by its PV
        if (sc.g >= NS) ok = mbar_wait(&o_full[s_buf], s_ph ^ 1, err, 0x2d);
        if (ok && sc.j == 0) ok = mbar_wait(&q_full[sc.k & 1], (sc.k >> 1) & 1, err, 0x23);
        ok = ok && mbar_wait(&k_full[k_st], k_ph, err, 0x24);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = q_lo0 + (sc.k & 1) * QD, b = k_lo0 + k_st * KVD;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t o = (kk >> 2) * PD + (kk & 3) * 2;
          mma_ss(tmem_base + s_buf * 128, a + o, b + o, DHI, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[s_buf]);
        if (++s_buf == NS) s_buf = 0, s_ph ^= 1;
        if (++k_st == KST) k_st = 0, k_ph ^= 1;
      }
    } else if (warp == 1 && lane == 0 && nunits > 0) {
      constexpr uint32_t idesc_o = umma_idesc_bf16(128, DH, 0, 1);  // V is MN-major
      const uint32_t v_lo0 = (smem_u32(sV) >> 4) | (PD << 16);     // LBO one panel (MN-major)
      AttnCursor pc;
      pc.init(nunits, B, Tq, Tk, H, Hkv);
      bool ok = true;
      uint32_t p_buf = 0, p_ph = 0, v_st = 0;
      for (; ok && pc.valid(); pc.advance()) {
        ok = mbar_wait(&pv_ready[p_buf], p_ph, err, 0x25);
        // a unit's first PV overwrites O: the previous unit's O must have been read out
        if (ok && pc.j == 0 && pc.k > 0) ok = mbar_wait(o_free, (pc.k - 1) & 1, err, 0x27);
        if (!ok) break;
        tc_fence_after();
        const uint32_t b = v_lo0 + v_st * KVD;
#pragma unroll
        for (int kk = 0; kk < C::BKV / 16; ++kk) {
          // P: keys 16kk.. sit in 8 TMEM columns of their half (keys 64 hf + 2c, +1 in
          // column 64 hf + c). V: 16 keys = 16 rows of 128 B (kk * 128 in 16-byte
          // units); the next 64 head dims are one panel further (the LBO).
          mma_ts(tmem_base + C::O_COL, tmem_base + p_buf * 128 + (kk >> 2) * 64 + (kk & 3) * 8,
                 b + kk * 128, DHI, idesc_o, (pc.j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&o_full[p_buf]);
        if (++p_buf == NS) p_buf = 0, p_ph ^= 1;
        if (++v_st == VST) v_st = 0;
      }
      umma_commit(drain);
      mbar_wait(drain, 0, err, 0x28);
    }
  } else if (warp <= 9) {
    // ---------------- softmax / correction: warps 2..5 keys 0..63, 6..9 keys 64..127
    const int hf = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t t_o = lane_base + C::O_COL + hf * (DH / 2);
    float* xmax = xch;            // [step % 2][half][row]
    float* xsum = xch + 4 * 128;  // [unit % 2][half][row]
    bool ok = true;
    // PV(g) is waited on through o_full[g % NS]. A parity wait reads the right phase
    // only while its barrier is at most one phase ahead: the phase before (PV(g-NS))
    // has completed whenever this is asked (the score tile this thread last waited
    // for, S(g) or S(g+1), was issued behind it), and the phase after (PV(g+NS))
    // cannot complete before this thread releases P(g+NS).
    auto pv_wait = [&](int g, int site) {
      if (ok) ok = mbar_wait_warp(&o_full[g % NS], (g / NS) & 1, err, site);
    };
    // Every step and every unit end runs (and passes its barriers) even after a
    // timed-out wait, so the softmax warps always meet the same barriers.
    int g = 0;
    for (int k = 0; k < nunits; ++k) {
      const AttnUnit u = attn_unit(attn_unit_index(k, blockIdx.x, G), B, Tq, Tk, H, Hkv);
      const int qp = off + u.q0 + r;  // this row's position
      float m_ref = -INFINITY, l_run = 0.f;
      for (int j = 0; j < u.n; ++j, ++g) {
        const int buf = g % NS;
        if (ok) ok = mbar_wait_warp(&s_full[buf], (g / NS) & 1, err, 0x29);
        tc_fence_after();
        const uint32_t t_s = lane_base + buf * 128 + hf * 64;
        const int k0 = j * C::BKV + hf * 64;  // first key of this half
        float s[2][32];
        tmem_ld32(t_s, s[0]);
        tmem_ld32(t_s + 32, s[1]);
        tmem_wait_ld();
        if (k0 + 63 > off + u.q0) {  // some key of this half lies above some row's diagonal
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (k0 + c * 32 + i > qp) s[c][i] = -INFINITY;
        }
        // partial row max of the raw scores (the scale is positive), three at a time in
        // eight independent chains
        float m8[8];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int q = 0; q < 4; ++q) m8[4 * c + q] = fmaxf(s[c][2 * q], s[c][2 * q + 1]);
#pragma unroll
          for (int i = 8; i < 32; i += 8)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              m8[4 * c + q] = max3(m8[4 * c + q], s[c][i + 2 * q], s[c][i + 2 * q + 1]);
        }
        const float pm =
            max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        xmax[((g & 1) * 2 + hf) * 128 + r] = pm;
        quarter_bar(quarter);
        const float mx = fmaxf(pm, xmax[((g & 1) * 2 + (hf ^ 1)) * 128 + r]) * scale_log2;
        // Move the reference max only when this row's max grew by more than 2^8
        // (always on a unit's first step, where the reference is still -inf; key 0 is
        // visible to every row, so that step's max is finite). Both halves of a row
        // take the same decision from the same two partial maxima.
        const bool move = mx > m_ref + kRescaleLog2;
        const float m_new = move ? mx : m_ref;
        const float alpha = move ? ex2_approx(m_ref - m_new) : 1.f;  // 0 on the first step
        // p = 2^(s * scale - m): one FMA per key, the partial row sum in two
        // accumulators. P is packed in place as bf16 pairs (word k of chunk c: keys
        // 32c + 2k, 32c + 2k + 1) and stored over this half's first 32 score columns
        // (chunk c at column 16c, whose scores are already in registers).
        // The exponent arguments and the row sum use paired fp32 operations (one
        // instruction per two keys).
        const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_new, -m_new);
        float2 rs = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 x = __ffma2_rn(make_float2(s[c][i], s[c][i + 1]), sc2, nm2);
            const float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            rs = __fadd2_rn(rs, p);
            s[c][i >> 1] = __uint_as_float(pack_bf16x2(p.x, p.y));
          }
          tmem_st16(t_s + c * 16, *reinterpret_cast<const uint32_t(*)[16]>(s[c]));
        }
        l_run = l_run * alpha + (rs.x + rs.y);
        m_ref = m_new;
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          // Rescale this half of O once it holds PV(g-1); PV(g) is only issued after
          // this step's P is released.
          pv_wait(g - 1, 0x2a);
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < DH / 64; ++c) {
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
        if (lane == 0 && ok) mbar_arrive(&pv_ready[buf]);
      }
      // ---- unit end: hand the half row sum to the epilogue warps (slot k % 2, free
      // once they have read unit k - 2's) and go on with the next unit at once
      if (k >= 2 && ok) ok = mbar_wait_warp(&xsum_free[k & 1], ((k >> 1) & 1) ^ 1, err, 0x2e);
      xsum[((k & 1) * 2 + hf) * 128 + r] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(&l_ready[k & 1]);
    }
  } else {
    // ---------------- epilogue: warps 11..14, one output row per thread. For each unit:
    // wait for its last PV, read O out of TMEM (then O is free for the next unit's PVs),
    // normalise by the row sum, write the row into the unit's Q buffer (its last QK^T
    // has completed) in the 128-byte swizzled panel layout of the output tensor map,
    // and store the tile with TMA; rows past T_q are dropped by the store. The Q buffer
    // goes back to the producer once the store has read it.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t t_o = tmem_base + ((uint32_t)(quarter * 32) << 16) + C::O_COL;
    const float* xsum = xch + 4 * 128;
    const bool storer = warp == 11 && lane == 0;
    bool ok = true;
    int g = 0;
    for (int k = 0; k < nunits; ++k) {
      const AttnUnit u = attn_unit(attn_unit_index(k, blockIdx.x, G), B, Tq, Tk, H, Hkv);
      g += u.n;  // g - 1: the unit's last step
      if (ok) ok = mbar_wait_warp(&l_ready[k & 1], (k >> 1) & 1, err, 0x2f);
      const float inv_l = 1.f / (xsum[((k & 1) * 2) * 128 + r] + xsum[((k & 1) * 2 + 1) * 128 + r]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&xsum_free[k & 1]);
      // PV(g-1) via o_full[(g-1) % NS]: the phase before (PV(g-4)) completed before the
      // softmax could see S(g-1), and the phase after needs O released below.
      if (ok) ok = mbar_wait_warp(&o_full[(g - 1) % NS], ((g - 1) / NS) & 1, err, 0x2b);
      tc_fence_after();
      uint8_t* stage = sQ + (k & 1) * C::Q_BYTES;
#pragma unroll 1
      for (int c = 0; c < DH / 32; ++c) {
        float o[32];
        tmem_ld32(t_o + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = c * 32 + q * 8;
          const int p = col >> 6, ch = (col & 63) >> 3;
          uint4 w;
          w.x = pack_bf16x2(o[q * 8 + 0] * inv_l, o[q * 8 + 1] * inv_l);
          w.y = pack_bf16x2(o[q * 8 + 2] * inv_l, o[q * 8 + 3] * inv_l);
          w.z = pack_bf16x2(o[q * 8 + 4] * inv_l, o[q * 8 + 5] * inv_l);
          w.w = pack_bf16x2(o[q * 8 + 6] * inv_l, o[q * 8 + 7] * inv_l);
          *reinterpret_cast<uint4*>(stage + p * C::PANEL_BYTES + r * 128 + ((ch ^ (r & 7)) * 16)) = w;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);  // the next unit's PVs may overwrite O now
      fence_proxy_async_smem();  // generic-proxy writes, read next by the TMA engine
      epilogue_bar();
      if (storer) {
        if (ok) {
          for (int p = 0; p < C::PANELS; ++p)
            tma_store_3d(&tmO, stage + p * C::PANEL_BYTES, u.h * DH + p * 64, u.q0, u.b);
          bulk_commit_group();
          bulk_wait_group_read0();
          if (k + 2 < nunits) {  // the buffer is free: the Q of unit k + 2
            const AttnUnit u2 = attn_unit(attn_unit_index(k + 2, blockIdx.x, G), B, Tq, Tk, H, Hkv);
            mbar_arrive_expect_tx(&q_full[k & 1], C::Q_BYTES);
            for (int p = 0; p < C::PANELS; ++p)
              tma_load_3d(stage + p * C::PANEL_BYTES, &tmQ, &q_full[k & 1], p * 64, u2.q0,
                          u2.b * H + u2.h);
          }
        }
      }
    }
    if (storer) bulk_wait_group0();  // the last tile is written before the CTA exits
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
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_3d_bf16(&tq, q, (uint64_t)B * H, Tq, DH, (uint64_t)Tq * DH, 128) ||
      !make_tmap_3d_bf16(&tk, k, (uint64_t)B * Hkv, Tk, DH, (uint64_t)k_stride * DH, 128) ||
      !make_tmap_3d_bf16(&tv, v, (uint64_t)B * Hkv, Tk, DH, (uint64_t)k_stride * DH, 128) ||
      !make_tmap_3d_bf16(&to, o, (uint64_t)B, Tq, (uint64_t)H * DH, (uint64_t)Tq * H * DH, 128))
    return cudaErrorInvalidValue;
  auto kern = attn_tc_kernel<DH>;
  static std::atomic<unsigned long long> attr_done{0};
  if (cudaError_t e = ensure_smem_attr(kern, C::SMEM, attr_done); e != cudaSuccess)
    return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long units = (long long)((Tq + 127) / 128) * B * H;
  const int grid = units < sms ? (int)units : sms;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  return launch_k(kern, grid, kAttnTcThreads, C::SMEM, s, tq, tk, tv, to, B, Tq, Tk, H, Hkv,
                  scale_log2, err);
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
