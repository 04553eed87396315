// attn_sm100.cu -- warp-specialised tcgen05 quantized attention for B200.
//
// [SA1] "SageAttention: Accurate 8-Bit Attention for Plug-and-Play Inference
//       Acceleration", Algorithm 1 steps 3-9 and Eq. 4-5:
//         S_i^j = INT8_Matmul(Q_i, K_j^T) * delta_Q[i] * delta_K[j]
//         online softmax (m, l), O_i^j = rescale(O_i^{j-1}) + P~_i^j V_j
//         O_i = diag(l_i)^-1 O_i
// [SA2++] "SageAttention2++ ...", section "核心公式": the 8+8 P~V with
//       static delta_P = 1/448 and per-channel delta_V.
//
// One CTA owns two 128-row q tiles of one (batch, head) and streams the kv
// tiles of that head through a multi-stage TMA/mbarrier ring.  16 warps:
//   warps 0-3   softmax of q tile 0, warps 4-7 softmax of q tile 1: each
//               thread owns one row; it reads S from TMEM, keeps the running
//               max m and sum l in registers, hands the row's rescale factor
//               alpha = 2^(m_old - m_new) to the correction warps through
//               shared memory right after the row max (so the rescale of O
//               overlaps the exponentials), and writes P~: fp16 P~ back into
//               the TMEM columns of S (variant B), or e4m3 of 448 P~ into a
//               shared-memory tile (8+8).  In the 8+8 kernel S_g(j+1) is
//               computed while the softmax of S_g(j) runs: the softmax frees
//               the TMEM columns of S_g as soon as it has loaded them.
//   warps 8-11  correction: rescale the rows of O_g in TMEM by alpha before
//               the next P~V accumulates into them, and the epilogue
//               (O / l, x delta_v[c] / 448 for 8+8, fp16 store).
//   warp 15     MMA issuer (one thread): S_g = Q_g K_j^T (kind::i8, s32 in
//               TMEM), and for variant B also O_g += P_g V_j (kind::f16,
//               P_g from TMEM); it also allocates and frees the TMEM.
//   warp 13     TMA producer (Q once, then K_j, V_j per ring stage).
//   warp 14     8+8: P~V issuer (one thread): O_g += P_g V_j (kind::f8f6f4,
//               P_g from shared memory), apart from the S issuer so that
//               neither waits behind the other.
//   warp 12     idle (completes the last warpgroup for setmaxnreg).  Warp w
//               runs on sub-partition w % 4: the three helper roles sit on
//               sub-partitions 1-3 (measured slightly faster than 0-2).
// Registers: launched at 128 per thread; setmaxnreg then gives the softmax
// warpgroups 192 (B) or 184 (8+8), the correction warpgroup 56 / 72 and the
// last warpgroup 72 / 64, within the 16*128 per lane the launch provides.
// Tensor memory (512 columns x 128 lanes): S_0 [0,128), S_1 [128,256),
// O_0 [256,256+d), O_1 [384,384+d); variant B's P_g aliases the first
// columns of S_g.
// Every wait is bounded (see mbar_wait); on expiry the CTA records the
// error, abandons its work, drains its in-flight copies and MMAs, frees
// tensor memory and exits.
#include <cuda_fp16.h>
#include <math.h>

#include <cmath>
#include <stdio.h>

#include "sage_internal.h"

namespace sage {

constexpr int kBM = 128, kBN = 128;
constexpr int kMmaWarp = 15, kProducerWarp = 13;  // warps 8-11: correction
constexpr int kPvWarp = 14;  // 8+8: issues the P~V MMAs
constexpr int kAttnThreads = 512;
// setmaxnreg shares per role (softmax, correction, other warps); 8 x soft +
// 4 x corr + 4 x misc must not exceed 16 x 128 (the launch budget per lane).
template <int VAR> struct Regs;
template <> struct Regs<0> { static constexpr uint32_t soft = 192, corr = 56, misc = 72; };
template <> struct Regs<1> { static constexpr uint32_t soft = 184, corr = 72, misc = 64; };
static_assert(8 * Regs<0>::soft + 4 * Regs<0>::corr + 4 * Regs<0>::misc <= 16 * 128, "register split");
static_assert(8 * Regs<1>::soft + 4 * Regs<1>::corr + 4 * Regs<1>::misc <= 16 * 128, "register split");
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int VAR>
struct Cfg {
  static constexpr int NS = (VAR == 0 && D == 128) ? 3 : 4;  // ring stages
  static constexpr int Q_BYTES = kBM * D;
  static constexpr int K_BYTES = kBN * D;
  static constexpr int V_BYTES = kBN * D * (VAR == 0 ? 2 : 1);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_BYTES;
  // 8+8: P~ operand tiles in shared memory, one per q tile (K-major e4m3,
  // 128 rows of 128 keys, 128-byte swizzle)
  static constexpr bool PS = (VAR == 1);
  static constexpr int P_TILE = kBM * kBN;
  static constexpr int OFF_P = OFF_V + NS * V_BYTES;
  static constexpr int OFF_BAR = OFF_P + (PS ? 2 * P_TILE : 0);  // barriers, 512 B
  static constexpr int OFF_ALPHA = OFF_BAR + 512;            // float [2][128]
  static constexpr int OFF_L = OFF_ALPHA + 2 * 128 * 4;      // float [2][128]
  static constexpr int SMEM = OFF_L + 2 * 128 * 4 + 1024;    // + alignment slack
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
  __half* o;        // [B*H, N, D]
  int H, Hkv, N, nqb, nkvb;
  uint64_t timeout_ns;
  float log2_pr;    // 8+8: log2 of the P operand range (P operand = P_r * P~)
};

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
template <int VAR, bool MASKED>
__device__ __forceinline__ float tile_exp(uint32_t (&a)[128], float c, float bias, int lim) {
  const uint64_t c2 = pk2(c, c), b2 = pk2(bias, bias), magic2 = pk2(-12582912.f, -12582912.f);
  uint64_t sum2[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) sum2[t] = 0;
#pragma unroll
  for (int i = 0; i < 128; i += 4) {
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const uint64_t f2 = add2(pk2(__uint_as_float(a[i + e] + 0x4B400000u),
                                   __uint_as_float(a[i + e + 1] + 0x4B400000u)), magic2);
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

template <int D, int VAR, bool CAUSAL>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const AttnKParams p) {
  using C = Cfg<D, VAR>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  float* s_alpha = reinterpret_cast<float*>(smem + C::OFF_ALPHA);  // [2][128]
  float* s_l = reinterpret_cast<float*>(smem + C::OFF_L);          // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + NS;
  uint64_t* v_full = k_empty + NS;
  uint64_t* v_empty = v_full + NS;
  uint64_t* s_full = v_empty + NS;   // [2] S_g(j) in TMEM          (MMA commit)
  uint64_t* p_full = s_full + 2;     // [2] P_g(j) in TMEM          (128 softmax threads)
  uint64_t* a_full = p_full + 2;     // [2] alpha_g(j) in smem      (128 softmax threads)
  uint64_t* o_ready = a_full + 2;    // [2] O_g rescaled for j      (128 correction threads)
  uint64_t* pv_done = o_ready + 2;   // [2] PV_g(j) complete        (MMA commit)
  uint64_t* l_full = pv_done + 2;    // [2] final l_g in smem       (128 softmax threads)
  uint64_t* s_free = l_full + 2;     // [2] S_g(j) loaded by softmax (128 softmax threads; 8+8)
  uint64_t* mma_done = s_free + 2;
  uint64_t* pv_mma_done = mma_done + 1;  // end of the PV issuer's MMAs (8+8)
  // Parity waits are only sound if no waiter can fall two phases behind the
  // barrier.  8+8 protocol, per tile g and kv step j:
  //   s_full(j)  S_g(j+1) needs s_free(j), which the softmax arrives after
  //              waiting s_full(j).
  //   s_free(j)  the softmax arrives s_free(j+1) after s_full(j+1), which
  //              needs the S issuer to have waited s_free(j).
  //   p_full(j)  the softmax arrives p_full(j+1) after waiting pv_done(j),
  //              i.e. after the P~V issuer consumed p_full(j).
  //   pv_done(j) PV_g(j+1) needs p_full(j+1) (softmax past its pv_done(j)
  //              wait) and o_ready(j+1) (correction past its pv_done(j) wait).
  //   a_full(j)  the softmax arrives a_full(j+1) after pv_done(j), and PV_g(j)
  //              is issued only after o_ready(j): the correction has already
  //              consumed a_full(j) (and read alpha(j) from the shared slot).
  //   o_ready(j) o_ready(j+1) needs pv_done(j), so the P~V issuer has passed
  //              its o_ready(j) wait.
  //   v_full / v_empty, k_full / k_empty: the usual ring, one consumer each
  //              (the P~V issuer for V, the S issuer for K).
  // Variant B gets the same bounds from the order S_g(j+1) after PV_g(j)
  // (P~ lives in the columns of S).
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(pv_mma_done + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int npairs = gridDim.x;
  // causal: heaviest q-tile pairs first
  const int pp = CAUSAL ? (npairs - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
  const int bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;
  const int zkv = b * p.Hkv + h / (p.H / p.Hkv);
  const int qb0 = 2 * pp;
  const bool has1 = qb0 + 1 < p.nqb;
  const int nkv0 = CAUSAL ? min(qb0 + 1, p.nkvb) : p.nkvb;
  const int nkv1 = CAUSAL ? min(qb0 + 2, p.nkvb) : p.nkvb;
  const int nkv = has1 ? nkv1 : nkv0;
  const uint64_t tlim = p.timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&p_full[g], 128);
      mbar_init(&a_full[g], 128);
      mbar_init(&o_ready[g], 128);
      mbar_init(&pv_done[g], 1);
      mbar_init(&l_full[g], 128);
      mbar_init(&s_free[g], 128);
    }
    mbar_init(mma_done, 1);
    mbar_init(pv_mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
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
    const int qb = qb0 + g;
    if (g == 0 || has1) {
      const int nkv_g = g == 0 ? nkv0 : nkv1;
      const uint32_t tS = tmem + (static_cast<uint32_t>(wq * 32) << 16) + g * 128;
      const uint32_t sP_g = smem_u32(smem + C::OFF_P) + g * C::P_TILE;
      const float dq_l2e = __fmul_rn(p.dq[static_cast<size_t>(bh) * p.nqb + qb], kLog2e);
      const float* dkp = p.dk + static_cast<size_t>(zkv) * p.nkvb;
      float m = -INFINITY, l = 0.f;
      float dk_next = dkp[0];
      for (int j = 0; j < nkv_g; ++j) {
        const float c = __fmul_rn(dq_l2e, dk_next);
        if (j + 1 < nkv_g) dk_next = dkp[j + 1];
        // tcgen05.ld/st below are warp-collective: every lane takes the same branch
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&s_full[g], j & 1, s_abort, tlim, 8))) break;
        tc_fence_after();
        uint32_t a[128];
        SAGE_TMEM_LD32(tS + 0, a);
        SAGE_TMEM_LD32(tS + 32, (a + 32));
        SAGE_TMEM_LD32(tS + 64, (a + 64));
        SAGE_TMEM_LD32(tS + 96, (a + 96));
        tmem_wait_ld();
        if (C::PS) {  // S_g's columns may now take S_g(j+1)
          tc_fence_before();
          mbar_arrive(&s_free[g]);
        }
        const int valid = p.N - j * kBN;  // keys left in this tile
        const bool masked = (CAUSAL && j == qb) || valid < kBN;
        const int lim = masked ? min(valid, (CAUSAL && j == qb) ? r + 1 : kBN) : kBN;
        const int imax = masked ? tile_rowmax<true>(a, lim) : tile_rowmax<false>(a, lim);
        // |imax| <= d * 127^2 < 2^22: the int -> float conversion is exact.
        const float m_new = fmaxf(m, __fmul_rn(static_cast<float>(imax), c));
        const float alpha = ex2_approx(m - m_new);  // 0 on the first tile
        if (j > 0) {
          // the correction warps rescale O_g while this thread computes P~.
          // 8+8: wait for PV_g(j-1) first; it is issued only once O_g was
          // rescaled for j-1 (so the alpha slot is free), and it frees the P
          // tile.  Variant B: S_g(j) was issued after PV_g(j-1), so both
          // already hold.
          if (C::PS && !__all_sync(0xFFFFFFFFu, mbar_wait(&pv_done[g], (j - 1) & 1, s_abort, tlim, 15)))
            break;
          s_alpha[g * 128 + r] = alpha;
          mbar_arrive(&a_full[g]);
        }
        const float bias = (VAR == 1) ? (p.log2_pr - m_new) : -m_new;
        const float rs = masked ? tile_exp<VAR, true>(a, c, bias, lim) : tile_exp<VAR, false>(a, c, bias, lim);
        l = __fmaf_rn(alpha, l, rs);
        if (C::PS) {
          // row r, 16-byte chunk c (keys 16c..16c+15) at the 128-byte-swizzled
          // position of the K-major operand layout
          const uint32_t rowp = sP_g + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(rowp + ((c ^ (r & 7)) << 4), a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
          fence_proxy_async_smem();
        } else {
          SAGE_TMEM_ST32(tS + 0, a);
          SAGE_TMEM_ST32(tS + 32, (a + 32));
          tmem_wait_st();
          tc_fence_before();
        }
        mbar_arrive(&p_full[g]);
        m = m_new;
      }
      s_l[g * 128 + r] = l;
      mbar_arrive(&l_full[g]);
    }
  } else if (warp < 12) {
    // ---------------------------------------------------------------- correction + epilogue
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Regs<VAR>::corr));
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    bool ok = true;
    // rescale of O_g for step j (j >= 1), in the order the MMA issuer consumes them
    for (int j = 1; ok && j < nkv; ++j) {
      for (int g = 0; g < 2; ++g) {
        if (g == 0 ? (j >= nkv0) : (!has1 || j >= nkv1)) continue;
        // O_g must hold the complete PV_g(j-1).  Variant B: implied by the
        // softmax having seen S_g(j), issued after PV_g(j-1).  8+8: wait.
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&a_full[g], (j - 1) & 1, s_abort, tlim, 10) &&
                                         (!C::PS || mbar_wait(&pv_done[g], (j - 1) & 1, s_abort, tlim, 14)))) {
          ok = false;
          break;
        }
        const float alpha = s_alpha[g * 128 + r];
        // O_g holds PV_g(j-1), complete
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
        tc_fence_before();
        mbar_arrive(&o_ready[g]);
      }
    }
    // epilogue: O / l (x delta_v[c] / 448 for 8+8, folded into l), fp16 rows
    for (int g = 0; ok && g < 2; ++g) {
      if (g == 1 && !has1) break;
      const int nkv_g = g == 0 ? nkv0 : nkv1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&l_full[g], 0, s_abort, tlim, 11) &&
                                       mbar_wait(&pv_done[g], (nkv_g - 1) & 1, s_abort, tlim, 9)))
        break;
      tc_fence_after();
      const float inv = 1.f / s_l[g * 128 + r];
      const int row = (qb0 + g) * kBM + r;
      const uint32_t tO = tmem + lane_off + 256 + g * 128;
      uint4* orow = reinterpret_cast<uint4*>(p.o + (static_cast<size_t>(bh) * p.N + row) * D);
      const float* dvp = p.dv + static_cast<size_t>(zkv) * D;
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
        if (row < p.N) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            orow[cb * 4 + i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Regs<VAR>::misc));
    if (warp == kMmaWarp && lane == 0) {
      // Variant B, issue order per kv step i (two q tiles ping-pong on the
      // tensor core):
      //   S_0(i), PV_1(i-1), S_1(i), PV_0(i)
      // so softmax 0 of step i overlaps PV_1(i-1) + S_1(i) and softmax 1
      // overlaps PV_0(i) + S_0(i+1).  S_g(i+1) overwrites the TMEM columns
      // that PV_g(i) reads P_g from; tcgen05.mma ops issued by one thread
      // execute in order, so the read precedes the overwrite.
      // The correction warps wait for pv_done_g before touching O_g.
      const uint64_t dQ0 = sdesc(smem_u32(sQ), 16, C::QK_SBO, C::QK_SW);
      const uint64_t dK0 = sdesc(smem_u32(sK), 16, C::QK_SBO, C::QK_SW);
      const uint64_t dV0 = sdesc(smem_u32(sV), C::V_LBO, C::V_SBO, C::V_SW);
      int k_seen = -1, v_seen = -1;
      auto active = [&](int g, int j) { return g == 0 ? (j < nkv0) : (has1 && j < nkv1); };
      auto issue_s = [&](int g, int j) -> bool {
        if (!active(g, j)) return true;
        // 8+8: S_g(j) reuses the columns of S_g(j-1) once the softmax has loaded them
        if (C::PS && j > 0 && !mbar_wait(&s_free[g], (j - 1) & 1, s_abort, tlim, 5)) return false;
        if (k_seen < j) {
          if (!mbar_wait(&k_full[j % NS], (j / NS) & 1, s_abort, tlim, 4)) return false;
          k_seen = j;
        }
        tc_fence_after();
        const uint64_t ad = dQ0 + (g * C::Q_BYTES >> 4);
        const uint64_t bd = dK0 + ((j % NS) * C::K_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8_ss(tmem + g * 128, ad + kk * 2, bd + kk * 2, C::IDESC_QK, kk > 0 ? 1u : 0u);
        tc_commit(&s_full[g]);
        return true;
      };
      auto issue_pv = [&](int g, int j) -> bool {  // variant B (P_g from TMEM)
        if (!active(g, j)) return true;
        if (v_seen < j) {
          if (!mbar_wait(&v_full[j % NS], (j / NS) & 1, s_abort, tlim, 6)) return false;
          v_seen = j;
        }
        if (!mbar_wait(&p_full[g], j & 1, s_abort, tlim, 7)) return false;
        if (j > 0 && !mbar_wait(&o_ready[g], (j - 1) & 1, s_abort, tlim, 12)) return false;
        tc_fence_after();
        const uint64_t vd = dV0 + ((j % NS) * C::V_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / C::PV_K; ++kk) {
          const uint64_t bd = vd + (kk * C::PV_K * C::V_ROW >> 4);
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          mma_f16_ts(tmem + 256 + g * 128, tmem + g * 128 + kk * 8, bd, C::IDESC_PV, acc);
        }
        tc_commit(&pv_done[g]);
        return true;
      };
      bool ok = mbar_wait(bar_q, 0, s_abort, tlim, 3);
      ok = ok && issue_s(0, 0) && issue_s(1, 0);
      if (ok) tc_commit(&k_empty[0]);
      if (C::PS) {
        // S_g(i+1) is issued as soon as the softmax has loaded S_g(i), so it
        // is ready when the softmax of step i ends; the P~V MMAs come from
        // their own issuer (warp kPvWarp), so neither waits behind the other.
        // The two streams touch disjoint TMEM (S vs O) and shared memory.
        for (int i = 0; ok && i + 1 < nkv; ++i) {
          ok = issue_s(0, i + 1) && issue_s(1, i + 1);
          if (!ok) break;
          tc_commit(&k_empty[(i + 1) % NS]);
        }
      } else {
        ok = ok && issue_pv(0, 0);
        for (int i = 1; ok && i < nkv; ++i) {
          ok = issue_s(0, i) && issue_pv(1, i - 1);
          if (!ok) break;
          tc_commit(&v_empty[(i - 1) % NS]);
          ok = issue_s(1, i);
          if (!ok) break;
          tc_commit(&k_empty[i % NS]);
          ok = issue_pv(0, i);
        }
        if (ok && issue_pv(1, nkv - 1)) tc_commit(&v_empty[(nkv - 1) % NS]);
      }
      tc_commit(mma_done);
      drain_wait(mma_done, 0, tlim);
    } else if (C::PS && warp == kPvWarp && lane == 0) {
      // 8+8 P~V issuer: PV_0(i), PV_1(i) per kv step, each once P_g(i) is in
      // shared memory and O_g has been rescaled for step i.
      const uint64_t dV0 = sdesc(smem_u32(sV), C::V_LBO, C::V_SBO, C::V_SW);
      const uint64_t dP0 = sdesc(smem_u32(smem + C::OFF_P), 16, 1024, SW_128B);
      bool ok = true;
      for (int i = 0; ok && i < nkv; ++i) {
        ok = mbar_wait(&v_full[i % NS], (i / NS) & 1, s_abort, tlim, 6);
        for (int g = 0; ok && g < 2; ++g) {
          if (!(g == 0 ? (i < nkv0) : (has1 && i < nkv1))) continue;
          ok = mbar_wait(&p_full[g], i & 1, s_abort, tlim, 7) &&
               (i == 0 || mbar_wait(&o_ready[g], (i - 1) & 1, s_abort, tlim, 12));
          if (!ok) break;
          tc_fence_after();
          const uint64_t vd = dV0 + ((i % NS) * C::V_BYTES >> 4);
#pragma unroll
          for (int kk = 0; kk < kBN / C::PV_K; ++kk)
            mma_f8_ss(tmem + 256 + g * 128, dP0 + (g * C::P_TILE >> 4) + kk * 2,
                      vd + (kk * C::PV_K * C::V_ROW >> 4), C::IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&pv_done[g]);
        }
        if (ok) tc_commit(&v_empty[i % NS]);
      }
      tc_commit(pv_mma_done);
      drain_wait(pv_mma_done, 0, tlim);
    } else if (warp == kProducerWarp && lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar_q, (has1 ? 2 : 1) * C::Q_BYTES);
      tma_load_3d(&tm_q, bar_q, sQ, 0, qb0 * kBM, bh);
      if (has1) tma_load_3d(&tm_q, bar_q, sQ + C::Q_BYTES, 0, (qb0 + 1) * kBM, bh);
      int nk = 0, nv = 0;  // loads issued
      for (int j = 0; j < nkv; ++j) {
        const int s = j % NS;
        const uint32_t ph = ((j / NS) & 1) ^ 1;
        if (!mbar_wait(&k_empty[s], ph, s_abort, tlim, 1)) break;
        mbar_arrive_expect_tx(&k_full[s], C::K_BYTES);
        tma_load_3d(&tm_k, &k_full[s], sK + s * C::K_BYTES, 0, j * kBN, zkv);
        ++nk;
        if (!mbar_wait(&v_empty[s], ph, s_abort, tlim, 2)) break;
        mbar_arrive_expect_tx(&v_full[s], C::V_BYTES);
        uint8_t* dst = sV + s * C::V_BYTES;
        if (VAR == 0 && D == 128) {
          tma_load_3d(&tm_v, &v_full[s], dst, 0, j * kBN, zkv);
          tma_load_3d(&tm_v, &v_full[s], dst + C::V_BOX_BYTES, 64, j * kBN, zkv);
        } else {
          tma_load_3d(&tm_v, &v_full[s], dst, 0, j * kBN, zkv);
        }
        ++nv;
      }
      if (*s_abort) {  // let the copies still in flight land before the CTA exits
        drain_wait(bar_q, 0, tlim);
        for (int i = max(0, nk - NS); i < nk; ++i) drain_wait(&k_full[i % NS], (i / NS) & 1, tlim);
        for (int i = max(0, nv - NS); i < nv; ++i) drain_wait(&v_full[i % NS], (i / NS) & 1, tlim);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D map over [slabs][N][d] of `elem`-byte elements, box = box_inner x 128 x 1.
static bool make_map_impl(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem, int d,
                     int N, int slabs, int box_inner, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
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

static bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem, int d,
                     int N, int slabs, int box_inner, CUtensorMapSwizzle sw) {
  if (encode_fn() == nullptr) {
    set_error_detail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorInvalidValue);
    return false;
  }
  return make_map_impl(m, base, dt, elem, d, N, slabs, box_inner, sw);
}

template <int D, int VAR, bool CAUSAL>
static cudaError_t launch_t(const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<D, VAR>;
  static bool attr_set = false;
  auto kern = k_attn<D, VAR, CAUSAL>;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) {
      set_error_detail("cudaFuncSetAttribute(attention)", e, C::SMEM);
      return e;
    }
    attr_set = true;
  }
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  bool ok = make_map(&tq, a.q_hat, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, a.N, a.B * a.H, D, qk_sw) &&
            make_map(&tk, a.k_hat, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, a.N, a.B * a.H_kv, D, qk_sw);
  if (VAR == 0)
    ok = ok && make_map(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, D, a.N, a.B * a.H_kv, 64,
                        CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_map(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, a.N, a.B * a.H_kv, D, qk_sw);
  if (!ok) return cudaErrorInvalidValue;
  AttnKParams kp;
  kp.dq = a.delta_q;
  kp.dk = a.delta_k;
  kp.dv = a.delta_v;
  kp.o = static_cast<__half*>(a.o);
  kp.H = a.H;
  kp.Hkv = a.H_kv;
  kp.N = a.N;
  kp.nqb = (a.N + kBM - 1) / kBM;
  kp.nkvb = (a.N + kBN - 1) / kBN;
  kp.timeout_ns = a.timeout_ns;
  kp.log2_pr = static_cast<float>(std::log2(static_cast<double>(a.p_r)));
  dim3 grid((kp.nqb + 1) / 2, a.B * a.H);
  kern<<<grid, kAttnThreads, C::SMEM, st>>>(tq, tk, tv, kp);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) set_error_detail("attention kernel launch", e, C::SMEM);
  return e;
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st) {
  const bool c = a.causal != 0;
  if (a.d == 128) {
    if (a.variant == 0) return c ? launch_t<128, 0, true>(a, st) : launch_t<128, 0, false>(a, st);
    return c ? launch_t<128, 1, true>(a, st) : launch_t<128, 1, false>(a, st);
  }
  if (a.variant == 0) return c ? launch_t<64, 0, true>(a, st) : launch_t<64, 0, false>(a, st);
  return c ? launch_t<64, 1, true>(a, st) : launch_t<64, 1, false>(a, st);
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
