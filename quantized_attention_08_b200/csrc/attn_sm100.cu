// attn_sm100.cu -- persistent, warp-specialised tcgen05 quantized attention for B200.
//
// [SA1] "SageAttention: Accurate 8-Bit Attention for Plug-and-Play Inference
//       Acceleration", Algorithm 1 steps 3-9 and Eq. 4-5:
//         S_i^j = INT8_Matmul(Q_i, K_j^T) * delta_Q[i] * delta_K[j]
//         online softmax (m, l), O_i^j = rescale(O_i^{j-1}) + P~_i^j V_j
//         O_i = diag(l_i)^-1 O_i
//       Step 3 runs the outer loop over Q blocks in parallel, one per SM:
//       here one CTA per SM walks a static list of work items.
// [SA2++] "SageAttention2++ ...", section "核心公式": the 8+8 P~V with
//       static delta_P = 1/448 and per-channel delta_V.
//
// Work item: two 128-row q tiles (a "pair") of one (batch, head).  The grid
// has one CTA per SM; CTA c takes items c, 2G-1-c, 2G+c, ... (a boustrophedon
// over rounds of G items), so that costs that fall along the list even out.
// Causal lists hold the pairs longest first across all heads (longest
// processing time first); non-causal lists keep the pairs of one head
// together so that its K/V tiles are shared through L2.  Barrier phases,
// the tensor-memory allocation and the K/V ring run on across items: the
// next item's Q tiles load while the current one computes, and its first S
// tiles are issued while the correction warps store the previous output.
//
// 16 warps:
//   warps 0-3   softmax of q tile 0, warps 4-7 softmax of q tile 1, one row
//               per thread: S from tensor memory, integer row max, alpha =
//               2^(m_old - m_new) handed to the correction warps, then P~ as
//               e4m3(448 P~) into a shared-memory operand tile (8+8) or fp16
//               P~ over the tensor-memory columns of S (variant B).
//   warps 8-11  correction: rescale the rows of O_g in tensor memory by alpha
//               before the next P~V accumulates into them, and the epilogue
//               (O / l, x delta_v[c] / 448 for 8+8, fp16 store).
//   warp 15     S issuer (one thread): S_g = Q_g K_j^T (kind::i8, s32 in
//               tensor memory); it also allocates and frees the tensor memory.
//               Variant B: it also issues O_g += P_g V_j (kind::f16, P_g from
//               tensor memory), interleaved with the S MMAs.
//   warp 14     8+8 P~V issuer (one thread): O_g += P_g V_j (kind::f8f6f4,
//               P_g from shared memory).
//   warp 13     TMA producer (Q per item, then K_j, V_j per ring stage).
//   warp 12     idle (completes the last warpgroup for setmaxnreg).
// 8+8 look-ahead: the softmax frees the columns of S_g as soon as it has
// loaded them, so S_g(j+1) is computed during the softmax of S_g(j).
// Variant B keeps P~ in the columns of S: S_g(j+1) follows P~V_g(j).
// Tensor memory (512 columns x 128 lanes): S_0 [0,128), S_1 [128,256),
// O_0 [256,256+d), O_1 [384,384+d).
// Every wait is bounded (see mbar_wait); on expiry the CTA records the
// error, abandons its work, drains its in-flight copies and MMAs, frees
// tensor memory and exits.
#include <cuda_fp16.h>
#include <math.h>

#include <atomic>
#include <cmath>
#include <stdio.h>

#include "sage_internal.h"

namespace sage {

constexpr int kBM = 128, kBN = 128;
constexpr int kSWarp = 15, kPvWarp = 14, kProducerWarp = 13;  // warps 8-11: correction
constexpr int kAttnThreads = 512;
// setmaxnreg shares per role (softmax, correction, other warps); 8 x soft +
// 4 x corr + 4 x misc must not exceed 16 x 128 (the launch budget per lane).
template <int VAR> struct Regs;
template <> struct Regs<0> { static constexpr uint32_t soft = 176, corr = 72, misc = 72; };
template <> struct Regs<1> { static constexpr uint32_t soft = 184, corr = 72, misc = 64; };
static_assert(8 * Regs<0>::soft + 4 * Regs<0>::corr + 4 * Regs<0>::misc <= 16 * 128, "register split");
static_assert(8 * Regs<1>::soft + 4 * Regs<1>::corr + 4 * Regs<1>::misc <= 16 * 128, "register split");
constexpr float kLog2e = 1.4426950408889634f;
// int32 bit pattern of the fp32 value 1.5 * 2^23: for |a| < 2^22 the int32
// sum kMagicBits + a reads as the fp32 value 1.5 * 2^23 + a, exactly.
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr float kMagic = 12582912.f;

template <int D, int VAR>
struct Cfg {
  static constexpr bool PS = (VAR == 1);        // P~ through shared memory (8+8)
  static constexpr int PB = 1;                  // P~ (and alpha) buffers per q tile
  static constexpr int LS = PB + 1;             // slots for the final row sums of an item
  static constexpr int NS = (D == 128) ? 3 : 4; // K/V ring stages
  static constexpr int QB = 2;                  // Q buffers: the next item's Q loads early
  static constexpr int Q_BYTES = kBM * D;
  static constexpr int K_BYTES = kBN * D;
  static constexpr int V_BYTES = kBN * D * (VAR == 0 ? 2 : 1);
  static constexpr int P_TILE = kBM * kBN;      // e4m3 P~ of one q tile, K-major
  static constexpr int OFF_Q = 0;               // [QB][2 tiles]
  static constexpr int OFF_K = OFF_Q + QB * 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_BYTES;
  static constexpr int OFF_P = OFF_V + NS * V_BYTES;
  static constexpr int OFF_BAR = OFF_P + (PS ? 2 * PB * P_TILE : 0);  // barriers, 1 KB
  static constexpr int OFF_ALPHA = OFF_BAR + 1024;                    // float [2][PB][128]
  static constexpr int OFF_L = OFF_ALPHA + 2 * PB * 128 * 4;          // float [LS][2][128]
  static constexpr int SMEM = OFF_L + LS * 2 * 128 * 4 + 1024;        // + alignment slack
  // Q_hat / K_hat: K-major int8 rows of D bytes, swizzle span = row length.
  static constexpr uint32_t QK_SW = (D == 128) ? SW_128B : SW_64B;
  static constexpr uint32_t QK_SBO = 8 * D;
  // V: MN-major (channels contiguous); fp16 V arrives as boxes of 64 channels.
  static constexpr uint32_t V_ROW = (VAR == 0) ? 128 : D;  // bytes per kv row in a box
  static constexpr uint32_t V_BOX_BYTES = kBN * V_ROW;
  static constexpr uint32_t V_SW = (V_ROW == 128) ? SW_128B : SW_64B;
  static constexpr uint32_t V_SBO = 8 * V_ROW;
  static constexpr uint32_t V_LBO = V_BOX_BYTES;
  static constexpr int PV_K = (VAR == 0) ? 16 : 32;  // kv rows per PV instruction
  static constexpr uint32_t IDESC_QK = idesc(CF_S32, AF_S8, AF_S8, 0, 0, kBN, kBM);
  static constexpr uint32_t IDESC_PV =
      idesc(CF_F32, VAR == 0 ? AF_F16 : AF_E4M3, VAR == 0 ? AF_F16 : AF_E4M3, 0, 1, D, kBM);
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct AttnKParams {
  const float* dq;  // [B*H, nqb]
  const float* dk;  // [B*Hkv, nkvb]
  const float* dv;  // [B*Hkv, D] (8+8)
  __half* o;        // [B*H, N, D], or packed [H, T, D]
  const int* cu;    // packed sequences: token offsets [B+1] (nullptr: fixed length N)
  int T;            // packed: total tokens (rows of each head)
  // N: the sequence length (packed: the longest allowed); nqb = nkvb blocks
  // and npairs pairs of q blocks per (batch, head) at that length
  int H, Hkv, N, nqb, nkvb, npairs, BH, items;
  uint64_t timeout_ns;
  float log2_pr;    // 8+8: log2 of the P operand range (P operand = P_r * P~)
};

// One work item: q tiles qb0 and qb0 + 1 (if it exists) of head bh.  n is
// the sequence's length; Q rows start at row y0 of TMA slab qz, K and V rows
// at row y0 of slab kvz; the output rows at orow0.  nkv == 0: nothing to do
// (a pair past the end of a short packed sequence).
struct Item {
  int bh, zkv, qb0, nkv0, nkv1, nkv, n, y0, qz, kvz;
  size_t orow0;
  bool has1;
};

template <bool CAUSAL, bool PACKED>
__device__ __forceinline__ Item make_item(const AttnKParams& p, int item) {
  Item it;
  int pair;
  if (CAUSAL) {  // longest first: pair npairs-1 of every head, then npairs-2, ...
    pair = p.npairs - 1 - item / p.BH;
    it.bh = item % p.BH;
  } else {       // head-major: the pairs of one head are neighbours in the list
    it.bh = item / p.npairs;
    pair = item % p.npairs;
  }
  const int b = it.bh / p.H, h = it.bh % p.H;
  const int hkv = h / (p.H / p.Hkv);
  it.zkv = b * p.Hkv + hkv;
  if (!PACKED) {
    it.n = p.N;
    it.y0 = 0;
    it.qz = it.bh;
    it.kvz = it.zkv;
    it.orow0 = static_cast<size_t>(it.bh) * p.N;
  } else {  // offsets clamped to the tensor, so malformed ones stay in bounds
    int a = p.cu[b], e = p.cu[b + 1];
    a = a < 0 ? 0 : (a > p.T ? p.T : a);
    e = e < a ? a : (e > p.T ? p.T : e);
    it.n = min(e - a, p.N);
    it.y0 = a;
    it.qz = h;
    it.kvz = hkv;
    it.orow0 = static_cast<size_t>(h) * p.T + a;
  }
  const int nb = (it.n + kBM - 1) / kBM;  // q blocks = kv tiles of this sequence
  it.qb0 = 2 * pair;
  it.has1 = it.qb0 + 1 < nb;
  it.nkv0 = CAUSAL ? min(it.qb0 + 1, nb) : nb;
  it.nkv1 = CAUSAL ? min(it.qb0 + 2, nb) : nb;
  it.nkv = (!PACKED || it.qb0 < nb) ? (it.has1 ? it.nkv1 : it.nkv0) : 0;
  return it;
}

// Item of round `rd` for this CTA, or -1 past the end: round rd covers
// items rd*G .. rd*G + G-1, walked forward in even rounds and backward in odd
// ones (a boustrophedon), so that costs that fall or rise along the list even
// out over the CTAs.
__device__ __forceinline__ int item_of_round(const AttnKParams& p, int rd) {
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const long long item = static_cast<long long>(rd) * G + ((rd & 1) ? (G - 1 - c) : c);
  return item < p.items ? static_cast<int>(item) : -1;
}

// Bounded wait that ignores the abort flag: used to drain in-flight work.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) {
      atomicOr(&g_error_word, ERR_TIMEOUT | (0xFFu << 8));
      return;
    }
  }
}

// ---------------------------------------------------------------- packed fp32 pairs
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 up2(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Row max of the s32 scores of one tile (columns >= lim masked when MASKED):
// eight independent 3-input chains, then a tree.
template <bool MASKED>
__device__ __forceinline__ int tile_rowmax(uint32_t (&a)[128], int lim) {
  if (MASKED) {
#pragma unroll
    for (int i = 0; i < 128; ++i)
      if (i >= lim) a[i] = 0x80000000u;
  }
  int mx[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    mx[t] = __vimax3_s32(static_cast<int>(a[16 * t]), static_cast<int>(a[16 * t + 1]),
                         static_cast<int>(a[16 * t + 2]));
#pragma unroll
    for (int i = 3; i < 15; i += 2)
      mx[t] = __vimax3_s32(mx[t], static_cast<int>(a[16 * t + i]), static_cast<int>(a[16 * t + i + 1]));
    mx[t] = max(mx[t], static_cast<int>(a[16 * t + 15]));
  }
  return max(__vimax3_s32(mx[0], mx[1], mx[2]), max(__vimax3_s32(mx[3], mx[4], mx[5]), max(mx[6], mx[7])));
}

// P~ of one tile for this thread's row: p = 2^(acc*c + bias) with
// c = delta_q * delta_k * log2(e), bias = -m_new (+ log2 P_r for 8+8).  `a`
// holds the s32 scores on entry and the packed P operand on exit (fp16x2, or
// 4 x e4m3 per word; lower columns in lower bits).  Returns the row sum of
// the unrounded P values.
template <int VAR, bool MASKED, bool CVT>
__device__ __forceinline__ float tile_exp(uint32_t (&a)[128], float c, float bias, int lim) {
  const uint64_t c2 = pk2(c, c), b2 = pk2(bias, bias), magic2 = pk2(-kMagic, -kMagic);
  uint64_t sum2[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) sum2[t] = 0;
#pragma unroll
  for (int i = 0; i < 128; i += 4) {
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      // acc as fp32, exactly (|acc| < 2^22): CVT, a plain conversion (ALU
      // pipe), else kMagicBits + acc, which reads as the fp32 value
      // 1.5 * 2^23 + acc, and one subtraction (FMA pipe); the kernel picks
      // the form measured faster for its variant and shape
      uint64_t f2;
      if (CVT) {
        f2 = pk2(static_cast<float>(static_cast<int>(a[i + e])), static_cast<float>(static_cast<int>(a[i + e + 1])));
      } else {
        f2 = add2(pk2(__uint_as_float(a[i + e] + kMagicBits), __uint_as_float(a[i + e + 1] + kMagicBits)), magic2);
      }
      const float2 x = up2(fma2(f2, c2, b2));
      p[e] = ex2_approx(x.x);
      p[e + 1] = ex2_approx(x.y);
      if (MASKED) {
        if (i + e >= lim) p[e] = 0.f;
        if (i + e + 1 >= lim) p[e + 1] = 0.f;
      }
    }
    sum2[(i / 4) & 3] = add2(sum2[(i / 4) & 3], add2(pk2(p[0], p[1]), pk2(p[2], p[3])));
    if (VAR == 0) {
      a[i / 2] = pack_f16x2(p[0], p[1]);
      a[i / 2 + 1] = pack_f16x2(p[2], p[3]);
    } else {
      a[i / 4] = pack_e4m3x2(p[0], p[1]) | (pack_e4m3x2(p[2], p[3]) << 16);
    }
  }
  const float2 s = up2(add2(add2(sum2[0], sum2[1]), add2(sum2[2], sum2[3])));
  return s.x + s.y;
}

template <int D, int VAR, bool CAUSAL, bool PACKED, bool CVT>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const AttnKParams p) {
  using C = Cfg<D, VAR>;
  constexpr int NS = C::NS, QB = C::QB, PB = C::PB, LS = C::LS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  float* s_alpha = reinterpret_cast<float*>(smem + C::OFF_ALPHA);  // [2][PB][128]
  float* s_l = reinterpret_cast<float*>(smem + C::OFF_L);          // [LS][2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q = bars;             // [QB] Q tiles of an item landed        (TMA)
  uint64_t* q_empty = bar_q + QB;     // [QB] last S MMA of an item done       (MMA commit)
  uint64_t* k_full = q_empty + QB;    // [NS]
  uint64_t* k_empty = k_full + NS;    // [NS]
  uint64_t* v_full = k_empty + NS;    // [NS]
  uint64_t* v_empty = v_full + NS;    // [NS]
  uint64_t* s_full = v_empty + NS;    // [2] S_g in tensor memory              (MMA commit)
  uint64_t* s_free = s_full + 2;      // [2] S_g loaded by the softmax (8+8)   (128 softmax threads)
  // per tile g and buffer b (kv step u uses buffer u % PB):
  uint64_t* p_full = s_free + 2;      // [2][PB] P_g written                   (128 softmax threads)
  uint64_t* a_full = p_full + 2 * PB; // [2][PB] alpha_g in shared memory      (128 softmax threads)
  uint64_t* pv_done = a_full + 2 * PB;  // [2][PB] P~V_g complete              (MMA commit)
  uint64_t* o_ready = pv_done + 2 * PB; // [2] O_g ready for the next P~V      (128 correction threads)
  uint64_t* l_full = o_ready + 2;     // [LS][2] final l_g of an item          (128 softmax threads)
  uint64_t* mma_done = l_full + 2 * LS;
  uint64_t* pv_mma_done = mma_done + 1;
  // Parity waits are only sound if no waiter can fall two phases behind the
  // barrier.  Per tile g, with u counting the kv steps of tile g over all
  // items of the CTA and b = u % PB the step's P~ / alpha buffer (the
  // arguments hold for any PB; one buffer per tile measured fastest, since
  // the softmax's wait for the previous P~V staggers the two tiles):
  //   s_full(u)   S_g(u+1) needs s_free(u+1), arrived by the softmax after
  //               its s_full(u) wait.  B: S_g(u+1) needs pv_done(u), which
  //               needs P_g(u), written after the s_full(u) wait.
  //   s_free(u)   one arrival before the first S (phase 0), then one per
  //               load: the next load needs the next S, issued only after
  //               the issuer waited this phase.
  //   p_full[b]   the softmax writes buffer b again (step u+PB) only after
  //               pv_done(u) (8+8) or s_full(u+1) (B): P~V_g(u) was issued,
  //               so the P~V issuer consumed p_full(u).
  //   a_full[b]   one arrival per step (unused alpha at an item's first
  //               step); step u+PB arrives after pv_done(u) (8+8) or
  //               s_full(u+1) (B); P~V_g(u) is issued after o_ready(u), i.e.
  //               after the correction consumed a_full(u) and alpha(u).
  //   pv_done[b]  P~V_g(u+PB) needs p_full(u+PB), written after the softmax's
  //               wait for pv_done(u); the correction's wait for pv_done(u-1)
  //               precedes its o_ready(u), which P~V_g(u) needs, and the
  //               epilogue's wait for an item's last step precedes the
  //               o_ready of the next item's first step.
  //   o_ready(u)  o_ready(u+1) follows the correction's pv_done(u) wait (or
  //               the epilogue, at an item's first step): the P~V issuer
  //               passed its o_ready(u) wait.
  //   l_full      PB + 1 slots by item: the softmax ends item i+PB+1 at a
  //               step u >= (last step of item i) + PB + 1, after its wait
  //               for pv_done(u-PB), which needs o_ready of a step of item
  //               i+1, which the correction arrives only after its epilogue
  //               of item i consumed that slot.
  //   bar_q, q_empty: one phase per item per buffer; a buffer is reloaded
  //               only after the last S of the item that used it.
  //   k/v full/empty: the usual ring, one consumer each.
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(pv_mma_done + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t tlim = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < QB; ++i) {
      mbar_init(&bar_q[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&s_free[g], 128);
      for (int b = 0; b < PB; ++b) {
        mbar_init(&p_full[g * PB + b], 128);
        mbar_init(&a_full[g * PB + b], 128);
        mbar_init(&pv_done[g * PB + b], 1);
      }
      mbar_init(&o_ready[g], 128);
      for (int sl = 0; sl < LS; ++sl) mbar_init(&l_full[sl * 2 + g], 128);
    }
    mbar_init(mma_done, 1);
    mbar_init(pv_mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kSWarp) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp < 8) {
    // ---------------------------------------------------------------- softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(Regs<VAR>::soft));
    const int g = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t tS = tmem + (static_cast<uint32_t>(wq * 32) << 16) + g * 128;
    const uint32_t sP_g = smem_u32(smem + C::OFF_P) + g * PB * C::P_TILE;
    if (C::PS) {
      tc_fence_before();
      mbar_arrive(&s_free[g]);  // phase 0: the first S_g may be issued
    }
    uint32_t u = 0, ul = 0;  // kv steps of tile g, items with tile g
    bool ok = true;
    for (int rd = 0; ok; ++rd) {
      const int item = item_of_round(p, rd);
      if (item < 0) break;
      const Item it = make_item<CAUSAL, PACKED>(p, item);
      if (PACKED && it.nkv == 0) continue;  // past the end of a short packed sequence
      if (g == 1 && !it.has1) continue;
      const int nkv_g = g == 0 ? it.nkv0 : it.nkv1;
      const int qb = it.qb0 + g;
      const float dq_l2e = __fmul_rn(p.dq[static_cast<size_t>(it.bh) * p.nqb + qb], kLog2e);
      const float* dkp = p.dk + static_cast<size_t>(it.zkv) * p.nkvb;
      float dk_next = dkp[0], m = -INFINITY, l = 0.f;
      for (int j = 0; j < nkv_g; ++j) {
        const float c = __fmul_rn(dq_l2e, dk_next);
        if (j + 1 < nkv_g) dk_next = dkp[j + 1];
        // tcgen05.ld/st below are warp-collective: every lane takes the same branch
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&s_full[g], u & 1, s_abort, tlim, 8))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t a[128];
        SAGE_TMEM_LD32(tS + 0, a);
        SAGE_TMEM_LD32(tS + 32, (a + 32));
        SAGE_TMEM_LD32(tS + 64, (a + 64));
        SAGE_TMEM_LD32(tS + 96, (a + 96));
        tmem_wait_ld();
        if (C::PS) {  // S_g's columns may now take S_g(u+1)
          tc_fence_before();
          mbar_arrive(&s_free[g]);
        }
        const int valid = it.n - j * kBN;  // keys left in this tile
        const bool masked = (CAUSAL && j == qb) || valid < kBN;
        const int lim = masked ? min(valid, (CAUSAL && j == qb) ? r + 1 : kBN) : kBN;
        const int imax = masked ? tile_rowmax<true>(a, lim) : tile_rowmax<false>(a, lim);
        // |imax| <= d * 127^2 < 2^22: the int -> float conversion is exact.
        const float m_new = fmaxf(m, __fmul_rn(static_cast<float>(imax), c));
        const float alpha = ex2_approx(m - m_new);  // 0 on the first tile
        // 8+8: the P tile and the alpha slot of buffer u % PB are free once
        // P~V_g(u-PB) is done (it is issued after the correction consumed
        // alpha(u-PB)).  B: S_g(u) ran after P~V_g(u-1), so both already hold.
        if (C::PS && u >= PB &&
            !__all_sync(0xFFFFFFFFu, mbar_wait(&pv_done[g * PB + u % PB], ((u - PB) / PB) & 1, s_abort,
                                               tlim, 15))) {
          ok = false;
          break;
        }
        // the correction warps rescale O_g while this thread computes P~
        // (at an item's first step alpha is 0 and unused: the hand-off keeps
        // one phase per step)
        s_alpha[(g * PB + u % PB) * 128 + r] = alpha;
        mbar_arrive(&a_full[g * PB + u % PB]);
        const float bias = (VAR == 1) ? (p.log2_pr - m_new) : -m_new;
        const float rs = masked ? tile_exp<VAR, true, CVT>(a, c, bias, lim) : tile_exp<VAR, false, CVT>(a, c, bias, lim);
        l = __fmaf_rn(alpha, l, rs);
        if (C::PS) {
          // row r, 16-byte chunk k (keys 16k..16k+15) at the 128-byte-swizzled
          // position of the K-major operand layout
          const uint32_t rowp = sP_g + (u % PB) * C::P_TILE + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            st_shared_v4(rowp + ((k ^ (r & 7)) << 4), a[4 * k], a[4 * k + 1], a[4 * k + 2], a[4 * k + 3]);
          fence_proxy_async_smem();
        } else {
          SAGE_TMEM_ST32(tS + 0, a);
          SAGE_TMEM_ST32(tS + 32, (a + 32));
          tmem_wait_st();
          tc_fence_before();
        }
        mbar_arrive(&p_full[g * PB + u % PB]);
        m = m_new;
        ++u;
        if (j == nkv_g - 1) {
          const int slot = static_cast<int>(ul % LS);
          s_l[(slot * 2 + g) * 128 + r] = l;
          mbar_arrive(&l_full[slot * 2 + g]);
          ++ul;
        }
      }
    }
  } else if (warp < 12) {
    // ---------------------------------------------------------------- correction + epilogue
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Regs<VAR>::corr));
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    uint32_t u[2] = {0, 0}, ul[2] = {0, 0};
    bool ok = true;
    for (int rd = 0; ok; ++rd) {
      const int item = item_of_round(p, rd);
      if (item < 0) break;
      const Item it = make_item<CAUSAL, PACKED>(p, item);
      if (PACKED && it.nkv == 0) continue;  // past the end of a short packed sequence
      // per kv step, in the order the P~V issuer consumes them: step 0 only
      // says that O_g is free (the previous item's epilogue read it), later
      // steps rescale O_g, which holds the complete P~V_g of the step before
      for (int j = 0; ok && j < it.nkv; ++j) {
        for (int g = 0; g < 2; ++g) {
          if (g == 0 ? (j >= it.nkv0) : (!it.has1 || j >= it.nkv1)) continue;
          const uint32_t b = u[g] % PB, bp = (u[g] + PB - 1) % PB;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&a_full[g * PB + b], (u[g] / PB) & 1, s_abort, tlim, 10) &&
                                           (j == 0 || mbar_wait(&pv_done[g * PB + bp], ((u[g] - 1) / PB) & 1,
                                                                s_abort, tlim, 14)))) {
            ok = false;
            break;
          }
          if (j > 0) {
            const float alpha = s_alpha[(g * PB + b) * 128 + r];
            if (__any_sync(0xFFFFFFFFu, alpha != 1.f)) {
              tc_fence_after();
              const uint32_t tO = tmem + lane_off + 256 + g * 128;
#pragma unroll 1
              for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t o[32];
                SAGE_TMEM_LD32(tO + cb * 32, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                SAGE_TMEM_ST32(tO + cb * 32, o);
              }
              tmem_wait_st();
            }
          }
          tc_fence_before();
          mbar_arrive(&o_ready[g]);
          ++u[g];
        }
      }
      // epilogue: O / l (x delta_v[c] / 448 for 8+8, folded into l), fp16 rows
      for (int g = 0; ok && g < 2; ++g) {
        if (g == 1 && !it.has1) break;
        const int slot = static_cast<int>(ul[g] % LS);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&l_full[slot * 2 + g], (ul[g] / LS) & 1, s_abort, tlim, 11) &&
                                         mbar_wait(&pv_done[g * PB + (u[g] - 1) % PB], ((u[g] - 1) / PB) & 1,
                                                   s_abort, tlim, 9))) {
          ok = false;
          break;
        }
        ++ul[g];
        tc_fence_after();
        const float inv = 1.f / s_l[(slot * 2 + g) * 128 + r];
        const int row = (it.qb0 + g) * kBM + r;
        const uint32_t tO = tmem + lane_off + 256 + g * 128;
        uint4* orow = reinterpret_cast<uint4*>(p.o + (it.orow0 + row) * D);
        const float* dvp = p.dv + static_cast<size_t>(it.zkv) * D;
#pragma unroll 1
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t o[32];
          SAGE_TMEM_LD32(tO + cb * 32, o);
          tmem_wait_ld();
          uint32_t hv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0 = __uint_as_float(o[2 * i]) * inv;
            float x1 = __uint_as_float(o[2 * i + 1]) * inv;
            if (VAR == 1) {
              x0 *= dvp[cb * 32 + 2 * i];
              x1 *= dvp[cb * 32 + 2 * i + 1];
            }
            hv[i] = pack_f16x2(x0, x1);
          }
          if (row < it.n) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              orow[cb * 4 + i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
          }
        }
        tc_fence_before();  // the next item's first P~V overwrites O_g
      }
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Regs<VAR>::misc));
    if (!C::PS && warp == kSWarp && lane == 0) {
      // Variant B: one thread issues both kinds of MMA, per item in the
      // order S_0(0), S_1(0), P~V_0(0), then per kv step i > 0
      //   S_0(i), P~V_1(i-1), S_1(i), P~V_0(i),
      // and P~V_1(last).  P~_g lives in the columns of S_g: tcgen05 MMAs
      // issued by one thread execute in order, so S_g(i) runs after
      // P~V_g(i-1) has read P~_g(i-1) without a round trip through a
      // barrier, and the two tiles keep the tensor core busy in turns.
      const uint64_t dQ0 = sdesc(smem_u32(sQ), 16, C::QK_SBO, C::QK_SW);
      const uint64_t dK0 = sdesc(smem_u32(sK), 16, C::QK_SBO, C::QK_SW);
      const uint64_t dV0 = sdesc(smem_u32(sV), C::V_LBO, C::V_SBO, C::V_SW);
      uint32_t kt = 0, itc = 0, us[2] = {0, 0}, up[2] = {0, 0};
      bool ok = true;
      for (int rd = 0; ok; ++rd) {
        const int item = item_of_round(p, rd);
        if (item < 0) break;
        const Item it = make_item<CAUSAL, PACKED>(p, item);
        if (PACKED && it.nkv == 0) continue;  // past the end of a short packed sequence
        const int qbuf = static_cast<int>(itc % QB);
        const uint32_t kt0 = kt;
        int k_seen = -1, v_seen = -1;
        auto active = [&](int g, int j) { return g == 0 ? (j < it.nkv0) : (it.has1 && j < it.nkv1); };
        auto issue_s = [&](int g, int j) -> bool {
          if (!active(g, j)) return true;
          const uint32_t st = kt0 + j;
          if (k_seen < j) {
            if (!mbar_wait(&k_full[st % NS], (st / NS) & 1, s_abort, tlim, 4)) return false;
            k_seen = j;
          }
          tc_fence_after();
          const uint64_t ad = dQ0 + ((qbuf * 2 + g) * C::Q_BYTES >> 4);
          const uint64_t bd = dK0 + ((st % NS) * C::K_BYTES >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_i8_ss(tmem + g * 128, ad + kk * 2, bd + kk * 2, C::IDESC_QK, kk > 0 ? 1u : 0u);
          tc_commit(&s_full[g]);
          ++us[g];
          return true;
        };
        auto issue_pv = [&](int g, int j) -> bool {
          if (!active(g, j)) return true;
          const uint32_t st = kt0 + j;
          if (v_seen < j) {
            if (!mbar_wait(&v_full[st % NS], (st / NS) & 1, s_abort, tlim, 6)) return false;
            v_seen = j;
          }
          if (!mbar_wait(&p_full[g], up[g] & 1, s_abort, tlim, 7) ||
              !mbar_wait(&o_ready[g], up[g] & 1, s_abort, tlim, 12))
            return false;
          tc_fence_after();
          const uint64_t vd = dV0 + ((st % NS) * C::V_BYTES >> 4);
#pragma unroll
          for (int kk = 0; kk < kBN / C::PV_K; ++kk)
            mma_f16_ts(tmem + 256 + g * 128, tmem + g * 128 + kk * 8, vd + (kk * C::PV_K * C::V_ROW >> 4),
                       C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&pv_done[g]);
          ++up[g];
          return true;
        };
        ok = mbar_wait(&bar_q[qbuf], (itc / QB) & 1, s_abort, tlim, 3) && issue_s(0, 0) && issue_s(1, 0);
        if (ok) tc_commit(&k_empty[kt0 % NS]);
        ok = ok && issue_pv(0, 0);
        for (int i = 1; ok && i < it.nkv; ++i) {
          ok = issue_s(0, i) && issue_pv(1, i - 1);
          if (!ok) break;
          tc_commit(&v_empty[(kt0 + i - 1) % NS]);
          ok = issue_s(1, i);
          if (!ok) break;
          tc_commit(&k_empty[(kt0 + i) % NS]);
          ok = issue_pv(0, i);
        }
        if (ok && issue_pv(1, it.nkv - 1)) {
          tc_commit(&v_empty[(kt0 + it.nkv - 1) % NS]);
          tc_commit(&q_empty[qbuf]);
        } else {
          ok = false;
        }
        kt += it.nkv;
        ++itc;
      }
      tc_commit(mma_done);
      drain_wait(mma_done, 0, tlim);
    } else if (C::PS && warp == kSWarp && lane == 0) {
      // 8+8 S issuer: S_0(j), S_1(j) per kv step of each item; S_g reuses
      // the columns of the previous S_g once the softmax has loaded it
      // (s_free), so S_g(j+1) runs during the softmax of S_g(j).
      const uint64_t dQ0 = sdesc(smem_u32(sQ), 16, C::QK_SBO, C::QK_SW);
      const uint64_t dK0 = sdesc(smem_u32(sK), 16, C::QK_SBO, C::QK_SW);
      uint32_t kt = 0, itc = 0, u[2] = {0, 0};
      bool ok = true;
      for (int rd = 0; ok; ++rd) {
        const int item = item_of_round(p, rd);
        if (item < 0) break;
        const Item it = make_item<CAUSAL, PACKED>(p, item);
        if (PACKED && it.nkv == 0) continue;  // past the end of a short packed sequence
        const int qbuf = static_cast<int>(itc % QB);
        ok = mbar_wait(&bar_q[qbuf], (itc / QB) & 1, s_abort, tlim, 3);
        for (int j = 0; ok && j < it.nkv; ++j) {
          const int s = static_cast<int>(kt % NS);
          ok = mbar_wait(&k_full[s], (kt / NS) & 1, s_abort, tlim, 4);
          for (int g = 0; ok && g < 2; ++g) {
            if (g == 0 ? (j >= it.nkv0) : (!it.has1 || j >= it.nkv1)) continue;
            ok = mbar_wait(&s_free[g], u[g] & 1, s_abort, tlim, 5);
            if (!ok) break;
            tc_fence_after();
            const uint64_t ad = dQ0 + ((qbuf * 2 + g) * C::Q_BYTES >> 4);
            const uint64_t bd = dK0 + (s * C::K_BYTES >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              mma_i8_ss(tmem + g * 128, ad + kk * 2, bd + kk * 2, C::IDESC_QK,
                        kk > 0 ? 1u : 0u);
            tc_commit(&s_full[g]);
            ++u[g];
          }
          if (!ok) break;
          tc_commit(&k_empty[s]);
          ++kt;
        }
        if (!ok) break;
        tc_commit(&q_empty[qbuf]);
        ++itc;
      }
      tc_commit(mma_done);
      drain_wait(mma_done, 0, tlim);
    } else if (C::PS && warp == kPvWarp && lane == 0) {
      // 8+8 P~V issuer: P~V_0(j), P~V_1(j) per kv step, each once P_g(j)
      // is in shared memory and O_g is ready for it (rescaled, or free at an
      // item's first step); apart from the S issuer so that neither waits
      // behind the other.
      const uint64_t dV0 = sdesc(smem_u32(sV), C::V_LBO, C::V_SBO, C::V_SW);
      const uint64_t dP0 = sdesc(smem_u32(smem + C::OFF_P), 16, 1024, SW_128B);
      uint32_t kt = 0, u[2] = {0, 0};
      bool ok = true;
      for (int rd = 0; ok; ++rd) {
        const int item = item_of_round(p, rd);
        if (item < 0) break;
        const Item it = make_item<CAUSAL, PACKED>(p, item);
        if (PACKED && it.nkv == 0) continue;  // past the end of a short packed sequence
        for (int j = 0; ok && j < it.nkv; ++j) {
          const int s = static_cast<int>(kt % NS);
          ok = mbar_wait(&v_full[s], (kt / NS) & 1, s_abort, tlim, 6);
          for (int g = 0; ok && g < 2; ++g) {
            if (g == 0 ? (j >= it.nkv0) : (!it.has1 || j >= it.nkv1)) continue;
            const uint32_t b = u[g] % PB;
            ok = mbar_wait(&p_full[g * PB + b], (u[g] / PB) & 1, s_abort, tlim, 7) &&
                 mbar_wait(&o_ready[g], u[g] & 1, s_abort, tlim, 12);
            if (!ok) break;
            tc_fence_after();
            const uint64_t vd = dV0 + (s * C::V_BYTES >> 4);
#pragma unroll
            for (int kk = 0; kk < kBN / C::PV_K; ++kk) {
              const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
              const uint64_t bd = vd + (kk * C::PV_K * C::V_ROW >> 4);
              mma_f8_ss(tmem + 256 + g * 128, dP0 + ((g * PB + b) * C::P_TILE >> 4) + kk * 2, bd,
                        C::IDESC_PV, acc);
            }
            tc_commit(&pv_done[g * PB + b]);
            ++u[g];
          }
          if (!ok) break;
          tc_commit(&v_empty[s]);
          ++kt;
        }
      }
      tc_commit(pv_mma_done);
      drain_wait(pv_mma_done, 0, tlim);
    } else if (warp == kProducerWarp && lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t nq = 0, nk = 0, nv = 0;  // loads issued
      bool ok = true;
      for (int rd = 0; ok; ++rd) {
        const int item = item_of_round(p, rd);
        if (item < 0) break;
        const Item it = make_item<CAUSAL, PACKED>(p, item);
        if (PACKED && it.nkv == 0) continue;  // past the end of a short packed sequence
        const int qbuf = static_cast<int>(nq % QB);
        if (!mbar_wait(&q_empty[qbuf], ((nq / QB) & 1) ^ 1, s_abort, tlim, 0)) break;
        mbar_arrive_expect_tx(&bar_q[qbuf], (it.has1 ? 2 : 1) * C::Q_BYTES);
        tma_load_3d(&tm_q, &bar_q[qbuf], sQ + (qbuf * 2) * C::Q_BYTES, 0, it.y0 + it.qb0 * kBM, it.qz);
        if (it.has1)
          tma_load_3d(&tm_q, &bar_q[qbuf], sQ + (qbuf * 2 + 1) * C::Q_BYTES, 0, it.y0 + (it.qb0 + 1) * kBM,
                      it.qz);
        ++nq;
        for (int j = 0; j < it.nkv; ++j) {
          const int s = static_cast<int>(nk % NS);
          if (!mbar_wait(&k_empty[s], ((nk / NS) & 1) ^ 1, s_abort, tlim, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[s], C::K_BYTES);
          tma_load_3d(&tm_k, &k_full[s], sK + s * C::K_BYTES, 0, it.y0 + j * kBN, it.kvz);
          ++nk;
          if (!mbar_wait(&v_empty[s], ((nv / NS) & 1) ^ 1, s_abort, tlim, 2)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&v_full[s], C::V_BYTES);
          uint8_t* dst = sV + s * C::V_BYTES;
          if (VAR == 0 && D == 128) {
            tma_load_3d(&tm_v, &v_full[s], dst, 0, it.y0 + j * kBN, it.kvz);
            tma_load_3d(&tm_v, &v_full[s], dst + C::V_BOX_BYTES, 64, it.y0 + j * kBN, it.kvz);
          } else {
            tma_load_3d(&tm_v, &v_full[s], dst, 0, it.y0 + j * kBN, it.kvz);
          }
          ++nv;
        }
      }
      if (*s_abort) {  // let the copies still in flight land before the CTA exits
        for (uint32_t i = nq > QB ? nq - QB : 0; i < nq; ++i) drain_wait(&bar_q[i % QB], (i / QB) & 1, tlim);
        for (uint32_t i = nk > NS ? nk - NS : 0; i < nk; ++i) drain_wait(&k_full[i % NS], (i / NS) & 1, tlim);
        for (uint32_t i = nv > NS ? nv - NS : 0; i < nv; ++i) drain_wait(&v_full[i % NS], (i / NS) & 1, tlim);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn lookup_encode_fn() {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(ptr);
  return nullptr;
}

static EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = lookup_encode_fn();  // thread-safe one-time initialisation
  return fn;
}

// 3-D map over [slabs][N][d] of `elem`-byte elements, box = box_inner x 128 x 1.
static bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem, int d, int N,
                     int slabs, int box_inner, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    set_error_detail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorInvalidValue);
    return false;
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(slabs)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem,
                                 static_cast<cuuint64_t>(N) * d * elem};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 128u, 1u};
  const cuuint32_t es[3] = {1u, 1u, 1u};
  const CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) set_error_detail("cuTensorMapEncodeTiled", cudaErrorInvalidValue, static_cast<int>(r));
  return r == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;

// Number of SMs of the current device (cached per device).
static cudaError_t sm_count(int* out) {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  *out = n;
  return cudaSuccess;
}

template <int D, int VAR, bool CAUSAL, bool PACKED, bool CVT>
static cudaError_t launch_t(const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<D, VAR>;
  // the dynamic shared-memory limit is a per-device function attribute
  static std::atomic<bool> attr_set[kMaxDevices];
  auto kern = k_attn<D, VAR, CAUSAL, PACKED, CVT>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) {
      set_error_detail("cudaFuncSetAttribute(attention)", e, C::SMEM);
      return e;
    }
    attr_set[dev].store(true, std::memory_order_release);
  }
  int sms = 0;
  if ((e = sm_count(&sms)) != cudaSuccess) return e;
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  // fixed layout: slabs of N rows, one per (batch, head); packed: one slab
  // of T rows per head
  const bool packed = PACKED;
  const int rows = packed ? a.T : a.N;
  const int qslabs = packed ? a.H : a.B * a.H, kvslabs = packed ? a.H_kv : a.B * a.H_kv;
  bool ok = make_map(&tq, a.q_hat, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, rows, qslabs, D, qk_sw) &&
            make_map(&tk, a.k_hat, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, rows, kvslabs, D, qk_sw);
  if (VAR == 0)
    ok = ok && make_map(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, D, rows, kvslabs, 64,
                        CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_map(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, rows, kvslabs, D, qk_sw);
  if (!ok) return cudaErrorInvalidValue;
  AttnKParams kp;
  kp.dq = a.delta_q;
  kp.dk = a.delta_k;
  kp.dv = a.delta_v;
  kp.o = static_cast<__half*>(a.o);
  kp.cu = a.cu;
  kp.T = a.T;
  kp.H = a.H;
  kp.Hkv = a.H_kv;
  kp.N = a.N;
  kp.nqb = (a.N + kBM - 1) / kBM;
  kp.nkvb = (a.N + kBN - 1) / kBN;
  kp.npairs = (kp.nqb + 1) / 2;
  kp.BH = a.B * a.H;
  const long long items = static_cast<long long>(kp.npairs) * kp.BH;
  if (items > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kp.items = static_cast<int>(items);
  kp.timeout_ns = a.timeout_ns;
  kp.log2_pr = static_cast<float>(std::log2(static_cast<double>(a.p_r)));
  // One persistent CTA per SM walks the item list (its prologue and epilogue
  // overlap the neighbouring items).  Long non-causal items (64 or more kv
  // tiles) are launched one CTA per item instead: there the prologue is
  // negligible, and the hardware's dynamic assignment of CTAs to SMs absorbs
  // the few-percent spread of per-SM speed that a fixed list cannot
  // (measured on the video-DiT shape).
  const bool persistent = CAUSAL || PACKED || kp.nkvb < 64;
  const int grid = persistent ? (kp.items < sms ? kp.items : sms) : kp.items;
  kern<<<grid, kAttnThreads, C::SMEM, st>>>(tq, tk, tv, kp);
  e = cudaGetLastError();
  if (e != cudaSuccess) set_error_detail("attention kernel launch", e, C::SMEM);
  return e;
}

// Score conversion (tile_exp's CVT) by measurement: the plain conversion
// for 8+8 at d = 128 and for 8+8 at d = 64 up to 8192 keys; the magic-number
// form for variant B and for longer d = 64 sequences.
template <bool PACKED>
static cudaError_t launch_p(const AttnArgs& a, cudaStream_t st) {
  const bool c = a.causal != 0;
  if (a.d == 128) {
    if (a.variant == 0)
      return c ? launch_t<128, 0, true, PACKED, false>(a, st) : launch_t<128, 0, false, PACKED, false>(a, st);
    return c ? launch_t<128, 1, true, PACKED, true>(a, st) : launch_t<128, 1, false, PACKED, true>(a, st);
  }
  if (a.variant == 0)
    return c ? launch_t<64, 0, true, PACKED, false>(a, st) : launch_t<64, 0, false, PACKED, false>(a, st);
  if (a.N <= 8192)
    return c ? launch_t<64, 1, true, PACKED, true>(a, st) : launch_t<64, 1, false, PACKED, true>(a, st);
  return c ? launch_t<64, 1, true, PACKED, false>(a, st) : launch_t<64, 1, false, PACKED, false>(a, st);
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st) {
  // packed sequences get their own instantiation: the per-sequence offsets
  // cost registers that the fixed-length kernel does not spend
  return a.cu != nullptr ? launch_p<true>(a, st) : launch_p<false>(a, st);
}

// ---------------------------------------------------------------- failure-detection self-test
__global__ void k_selftest_wait(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the bounded wait must give up
  if (threadIdx.x == 0) mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), timeout_ns, 0xEEu);
}

cudaError_t launch_selftest_wait(uint64_t timeout_ns, cudaStream_t st) {
  k_selftest_wait<<<1, 32, 0, st>>>(timeout_ns);
  return cudaGetLastError();
}

static thread_local char t_detail[256] = "none";

void set_error_detail(const char* step, cudaError_t e, int extra) {
  snprintf(t_detail, sizeof(t_detail), "%s: %s (%d) [%d]", step, cudaGetErrorString(e),
           static_cast<int>(e), extra);
}
const char* error_detail() { return t_detail; }

cudaError_t read_and_clear_error(uint32_t* word) {
  uint32_t w = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w));
  if (e != cudaSuccess) return e;
  if (w != 0) e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
  *word = w;
  return e;
}

}  // namespace sage
