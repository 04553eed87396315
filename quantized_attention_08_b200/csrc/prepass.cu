// prepass.cu -- Smooth K and the per-block quantizers, sm_100a.
//
// [SA1] "SageAttention: Accurate 8-Bit Attention for Plug-and-Play Inference
//       Acceleration", Algorithm 1 steps 1-2 and Eq. 6 (K <- K - mean(K);
//       psi_Q(Q/sqrt d), psi_K(K) per block).
// [SA2++] "SageAttention2++ ...", section "核心公式": delta = max|A|/127,
//       A_hat = round(A/delta); delta_V = colmax|V| / 448 (here / v_r).
//
// Three kernels, all HBM-bound:
//   k_colstats : per (slab, 256-token chunk) partial column statistics --
//                exact sums of K and the max |V| as fp16 magnitude bits.
//                Every fp16 value is an integer multiple of 2^-24 below 2^16,
//                so a sum of at most 256 of them needs 48 significant bits:
//                it is exact in fp64, and its value times 2^24 is stored as
//                an int64 (the chunk partials are then summed in int64).
//   k_finalize : per (slab, channel): mean_k = fp32(fp64(sum) * 2^-24 / N),
//                delta_v = fp32(colmax) / v_r.
//   k_quant    : one CTA per 128-token block of one head, for Q, K and V:
//                block absmax -> delta -> codes.
// With rotary tables, k_colstats_rope and k_quant_rope rotate each fp16 row
// of K (and Q) in registers first ([SA1] implementation detail 1: RoPE and
// the quantization in one pass, no rotated copy in HBM).  Their threads own
// both channels of every rotation pair (no shuffles), and one CTA serves
// several heads of the same tokens, so that each slice of the cos / sin
// tables is read once per head group rather than once per head.
// Every value is bit-identical to the definition whatever the grid, because
// the reductions are exact (integer sums, max) and each element's
// arithmetic is a fixed sequence of correctly rounded fp32 operations.
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <type_traits>

#include "quant_pair.cuh"
#include "sage_internal.h"

namespace sage {

constexpr int kStatRows = 256;  // tokens per statistics chunk
constexpr int kThreads = 256;

// Adds the two fp16 values packed in w to a pair of fp64 sums (exact: see
// the kernel notes above).
__device__ __forceinline__ void add_f16x2(double& lo, double& hi, uint32_t w) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
  lo = __dadd_rn(lo, static_cast<double>(f.x));
  hi = __dadd_rn(hi, static_cast<double>(f.y));
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float4 ld_f4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}

// Heads per CTA of the rotary kernels: the largest of 4, 2, 1 dividing the
// slab count per batch entry (so that a CTA's heads share their tokens).
inline int rope_group(int heads) { return heads % 4 == 0 ? 4 : heads % 2 == 0 ? 2 : 1; }

template <int D>
__global__ void __launch_bounds__(kThreads) k_colstats(const uint4* __restrict__ k,
                                                       const uint4* __restrict__ v, SeqLayout seq,
                                                       int Hkv, int nchunk, long long* __restrict__ ksum,
                                                       uint32_t* __restrict__ vmax) {
  constexpr int TPR = D / 8;             // threads per row: one uint4 (8 halves) each
  constexpr int RPI = kThreads / TPR;    // rows per iteration
  const int chunk = blockIdx.x, slab = blockIdx.y;
  const int cg = threadIdx.x % TPR, rl = threadIdx.x / TPR;
  size_t row0;
  int N;  // rows of this slab (token t of the sequence is row row0 + t)
  slab_rows(seq, slab, Hkv, &row0, &N);
  const int r0 = chunk * kStatRows, r1 = min(N, r0 + kStatRows);
  if (r0 >= N) return;  // a chunk past the end of a short sequence
  const size_t base = row0 * TPR + cg;

  double acc[8];
  uint32_t vm[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) { acc[e] = 0.0; vm[e] = 0; }

  // kUnroll rows per thread are loaded before any is reduced, so several
  // 16-byte loads per array are in flight; rows past the chunk read as +0,
  // which adds nothing to either statistic.
  constexpr int kUnroll = 4;
  for (int r = r0 + rl; r < r1; r += kUnroll * RPI) {
    uint4 xk[kUnroll], xv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int rr = r + u * RPI;
      const bool in = rr < r1;
      xk[u] = (k != nullptr && in) ? ld_stream(k + base + static_cast<size_t>(rr) * TPR) : make_uint4(0, 0, 0, 0);
      xv[u] = (v != nullptr && in) ? ld_stream(v + base + static_cast<size_t>(rr) * TPR) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (k != nullptr) {
        const uint32_t w[4] = {xk[u].x, xk[u].y, xk[u].z, xk[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) add_f16x2(acc[2 * e], acc[2 * e + 1], w[e]);
      }
      if (v != nullptr) {
        const uint32_t w[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          vm[2 * e] = max(vm[2 * e], w[e] & 0x7FFFu);          // |fp16| ordered as integer
          vm[2 * e + 1] = max(vm[2 * e + 1], (w[e] >> 16) & 0x7FFFu);
        }
      }
    }
  }

  __shared__ double s_sum[RPI][D];
  __shared__ uint32_t s_max[RPI][D];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    s_sum[rl][cg * 8 + e] = acc[e];
    s_max[rl][cg * 8 + e] = vm[e];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    double s = 0.0;
    uint32_t mx = 0;
#pragma unroll 4
    for (int i = 0; i < RPI; ++i) {
      s = __dadd_rn(s, s_sum[i][c]);
      mx = max(mx, s_max[i][c]);
    }
    const size_t o = (static_cast<size_t>(slab) * nchunk + chunk) * D + c;
    if (k != nullptr) ksum[o] = __double2ll_rn(__dmul_rn(s, 0x1p24));  // an integer: exact
    if (v != nullptr) vmax[o] = mx;
  }
}

// Rotary embedding, rotate-half pairing (channel i < D/2 pairs with
// i + D/2), of two channel pairs at once: wl holds fp16 x_i, x_i+1 of the
// lower half, wh their partners y, c / s the cos and sin of the two
// frequencies: lower y = fl(fl(x c) - fl(y s)), upper fl(fl(y c) + fl(x s)),
// each then rounded to fp16.
// The products are paired; the sums are scalar: ptxas contracts a paired
// product that feeds a paired add or sub into a fused multiply-add whatever
// the rounding qualifiers (and -fmad=false), which would round once instead
// of twice; scalar .rn adds are never contracted.
__device__ __forceinline__ void rope2(uint32_t& wl, uint32_t& wh, uint64_t c2, uint64_t s2) {
  const uint64_t x = f2_from_h2(wl), y = f2_from_h2(wh);
  const float2 xc = f2_unpack(f2_mul(x, c2)), ys = f2_unpack(f2_mul(y, s2));
  const float2 yc = f2_unpack(f2_mul(y, c2)), xs = f2_unpack(f2_mul(x, s2));
  const __half2 rl = __floats2half2_rn(__fsub_rn(xc.x, ys.x), __fsub_rn(xc.y, ys.y));
  const __half2 rh = __floats2half2_rn(__fadd_rn(yc.x, xs.x), __fadd_rn(yc.y, xs.y));
  wl = *reinterpret_cast<const uint32_t*>(&rl);
  wh = *reinterpret_cast<const uint32_t*>(&rh);
}

// Column statistics with rotary embedding: one CTA per (256-token chunk, G
// consecutive heads of one batch entry): exact sums of the rotated K and,
// if v is given (then G = 1), the max |V| as in k_colstats.  Rows outer,
// heads inner: a thread loads the cos / sin of its 8 frequencies at a
// token once and rotates that token's row in each of the G heads; U rows
// per thread are loaded before any is reduced.  Sums are exact (see
// k_colstats), so their order is free.
template <int D, int G, int U>
__global__ void __launch_bounds__(kThreads, 2) k_colstats_rope(const uint4* __restrict__ k,
                                                               const uint4* __restrict__ v, SeqLayout seq,
                                                               int Hkv, int nchunk,
                                                               long long* __restrict__ ksum,
                                                               uint32_t* __restrict__ vmax,
                                                               const float* __restrict__ cosT,
                                                               const float* __restrict__ sinT) {
  constexpr int TPR = D / 8, TP = TPR / 2, H2 = D / 2;
  constexpr int RPI = kThreads / TP;  // rows per iteration
  const int chunk = blockIdx.x, z0 = blockIdx.y * G;
  const int j = threadIdx.x % TP, rl = threadIdx.x / TP;
  size_t row0;
  int N = 0;
  slab_rows(seq, z0, Hkv, &row0, &N);  // head z0 + h starts h * T rows later (same tokens)
  const int r0 = chunk * kStatRows, r1 = min(N, r0 + kStatRows);
  if (r0 >= N) return;  // a chunk past the end of a short sequence
  const size_t hstride = static_cast<size_t>(seq.T) * TPR;
  const uint4* kb = k + row0 * TPR + j;
  const uint4* vb = v != nullptr ? v + row0 * TPR + j : nullptr;

  double acc[G][16];
  uint32_t vm[8];  // two fp16 magnitudes each: channels 8j+2e, +1 (e < 4), then the upper half
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[h][e] = 0.0;
#pragma unroll
  for (int e = 0; e < 8; ++e) vm[e] = 0;
#pragma unroll 1
  for (int r = r0 + rl; r < r1; r += U * RPI) {
    float4 tc[U][2], ts[U][2];
    uint4 lo[U][G], hi[U][G], vlo[U], vhi[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int rr = r + u * RPI;
      const bool in = rr < r1;
      const float* ct = cosT + static_cast<size_t>(in ? rr : r) * H2 + 8 * j;
      const float* st = sinT + static_cast<size_t>(in ? rr : r) * H2 + 8 * j;
      tc[u][0] = ld_f4(ct);
      tc[u][1] = ld_f4(ct + 4);
      ts[u][0] = ld_f4(st);
      ts[u][1] = ld_f4(st + 4);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const uint4* row = kb + h * hstride + static_cast<size_t>(rr) * TPR;
        lo[u][h] = in ? ld_stream(row) : make_uint4(0, 0, 0, 0);  // rows past the chunk add +0
        hi[u][h] = in ? ld_stream(row + TP) : make_uint4(0, 0, 0, 0);
      }
      if (vb != nullptr) {
        vlo[u] = in ? ld_stream(vb + static_cast<size_t>(rr) * TPR) : make_uint4(0, 0, 0, 0);
        vhi[u] = in ? ld_stream(vb + static_cast<size_t>(rr) * TPR + TP) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float4 c0 = tc[u][0], c1 = tc[u][1], s0 = ts[u][0], s1 = ts[u][1];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        uint4& l = lo[u][h];
        uint4& hh = hi[u][h];
        rope2(l.x, hh.x, f2_pack(c0.x, c0.y), f2_pack(s0.x, s0.y));
        rope2(l.y, hh.y, f2_pack(c0.z, c0.w), f2_pack(s0.z, s0.w));
        rope2(l.z, hh.z, f2_pack(c1.x, c1.y), f2_pack(s1.x, s1.y));
        rope2(l.w, hh.w, f2_pack(c1.z, c1.w), f2_pack(s1.z, s1.w));
        const uint32_t wl[4] = {l.x, l.y, l.z, l.w}, wh[4] = {hh.x, hh.y, hh.z, hh.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          add_f16x2(acc[h][2 * e], acc[h][2 * e + 1], wl[e]);
          add_f16x2(acc[h][8 + 2 * e], acc[h][8 + 2 * e + 1], wh[e]);
        }
      }
      if (vb != nullptr) {
        const uint32_t wl[4] = {vlo[u].x, vlo[u].y, vlo[u].z, vlo[u].w};
        const uint32_t wh[4] = {vhi[u].x, vhi[u].y, vhi[u].z, vhi[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // |fp16| ordered as integers, two per word
          vm[e] = __vmaxu2(vm[e], wl[e] & 0x7FFF7FFFu);
          vm[4 + e] = __vmaxu2(vm[4 + e], wh[e] & 0x7FFF7FFFu);
        }
      }
    }
  }
  // lanes of a warp with the same j hold the same channels: fold them, then
  // the warps through shared memory
#pragma unroll
  for (int o = TP; o < 32; o <<= 1) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[h][e] = __dadd_rn(acc[h][e], __shfl_xor_sync(0xFFFFFFFFu, acc[h][e], o));
#pragma unroll
    for (int e = 0; e < 8; ++e) vm[e] = __vmaxu2(vm[e], __shfl_xor_sync(0xFFFFFFFFu, vm[e], o));
  }
  __shared__ double s_sum[kThreads / 32][G][D];
  __shared__ uint32_t s_vm[kThreads / 32][D / 2];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < TP) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        s_sum[w][h][8 * j + e] = acc[h][e];
        s_sum[w][h][H2 + 8 * j + e] = acc[h][8 + e];
      }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s_vm[w][4 * j + e] = vm[e];
      s_vm[w][H2 / 2 + 4 * j + e] = vm[4 + e];
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < G * D; t += kThreads) {
    const int h = t / D, c = t % D;
    double sum = 0.0;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) sum = __dadd_rn(sum, s_sum[i][h][c]);
    ksum[(static_cast<size_t>(z0 + h) * nchunk + chunk) * D + c] = __double2ll_rn(__dmul_rn(sum, 0x1p24));
  }
  if (vb != nullptr && threadIdx.x < D) {
    const int c = threadIdx.x;
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) mx = max(mx, (s_vm[i][c >> 1] >> ((c & 1) * 16)) & 0xFFFFu);
    vmax[(static_cast<size_t>(z0) * nchunk + chunk) * D + c] = mx;
  }
}

// One CTA per (slab, 32 channels): its kFinWarps warps reduce interleaved
// chunks (lane = channel, several loads in flight per lane), then warp 0
// combines them.  Integer sums and maxima are exact, so the result does not
// depend on this order.
constexpr int kFinWarps = 16;
__global__ void __launch_bounds__(kFinWarps * 32) k_finalize(const long long* __restrict__ ksum,
                                                             const uint32_t* __restrict__ vmax, int nchunk_max,
                                                             int D, SeqLayout seq, int Hkv, float v_r,
                                                             float* __restrict__ mean_k, float* __restrict__ delta_v) {
  const int slab = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.y * 32 + lane;
  size_t row0;
  int N;
  slab_rows(seq, slab, Hkv, &row0, &N);
  const int nchunk = (N + kStatRows - 1) / kStatRows;  // chunks written for this slab
  __shared__ long long s_s[kFinWarps][32];
  __shared__ uint32_t s_m[kFinWarps][32];
  long long s = 0;
  uint32_t m = 0;
#pragma unroll 4
  for (int i = w; i < nchunk; i += kFinWarps) {
    const size_t o = (static_cast<size_t>(slab) * nchunk_max + i) * D + c;
    if (ksum != nullptr) s += ksum[o];
    if (vmax != nullptr) m = max(m, vmax[o]);
  }
  s_s[w][lane] = s;
  s_m[w][lane] = m;
  __syncthreads();
  if (w != 0) return;
#pragma unroll
  for (int i = 1; i < kFinWarps; ++i) {
    s += s_s[i][lane];
    m = max(m, s_m[i][lane]);
  }
  if (ksum != nullptr) {  // an empty sequence has mean 0
    const double sd = __dmul_rn(__ll2double_rn(s), 0x1p-24);
    mean_k[static_cast<size_t>(slab) * D + c] =
        N > 0 ? __double2float_rn(__ddiv_rn(sd, static_cast<double>(N))) : 0.f;
  }
  if (vmax != nullptr) {
    const float cm = __half2float(__ushort_as_half(static_cast<unsigned short>(m)));
    delta_v[static_cast<size_t>(slab) * D + c] = __fdiv_rn(cm, v_r);
  }
}

struct QuantJobs {
  const uint4* q;       // fp16 [B,H,N,D]
  const uint4* k;       // fp16 [B,Hkv,N,D]
  const uint4* v;       // fp16 [B,Hkv,N,D]
  uint2* q_hat;         // int8
  uint2* k_hat;
  uint2* v_hat;         // e4m3
  float* delta_q;       // [B,H,nb]
  float* delta_k;       // [B,Hkv,nb]
  const float* mean_k;  // [B,Hkv,D]
  const float* delta_v; // [B,Hkv,D]
  float sm_scale;
  const float* cos_t;   // rotary tables [N, D/2] or nullptr
  const float* sin_t;
  SeqLayout seq;        // rows of each slab
  int H, Hkv;           // heads of Q, of K and V (slab numbering)
  int nb;               // 128-token blocks per slab (the longest sequence's)
  int n_q, n_k, n_v;    // number of (slab, block) jobs of each kind
};

// E4M3 codes of one 128-token block of V (slab, blk): per-channel scale,
// no block reduction: e4m3(RN(v / delta_v[c])) (div_rn_by of quant_div.h,
// lane-wise), 0 for a channel whose delta_v is 0.
template <int D>
__device__ __forceinline__ void quant_v_block(const QuantJobs& J, int slab, int blk) {
  constexpr int TPR = D / 8;               // uint4 per token row
  constexpr int U = 128 * TPR / kThreads;  // uint4 per thread
  size_t srow;
  int len;
  slab_rows(J.seq, slab, J.Hkv, &srow, &len);
  const int rows = min(128, len - blk * 128);
  if (rows <= 0) return;  // a block past the end of a short sequence
  const size_t row0 = srow + static_cast<size_t>(blk) * 128;
  const uint4* src = J.v + row0 * TPR;
  uint2* dst = J.v_hat + row0 * TPR;
  const int cg = threadIdx.x % TPR;  // this thread's 8 channels: cg*8 .. cg*8+7 (fixed across u)
  uint4 raw[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int idx = threadIdx.x + kThreads * u;
    raw[u] = (idx / TPR < rows) ? ld_stream(src + idx) : make_uint4(0, 0, 0, 0);
  }
  uint64_t nd2[4], r2[4];
  uint32_t keep[4];  // per channel pair: byte masks of the channels with delta_v != 0
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float d0 = J.delta_v[static_cast<size_t>(slab) * D + cg * 8 + 2 * e];
    const float d1 = J.delta_v[static_cast<size_t>(slab) * D + cg * 8 + 2 * e + 1];
    nd2[e] = f2_pack(-d0, -d1);
    r2[e] = f2_pack(d0 != 0.f ? __frcp_rn(d0) : 0.f, d1 != 0.f ? __frcp_rn(d1) : 0.f);
    keep[e] = (d0 != 0.f ? 0x00FFu : 0u) | (d1 != 0.f ? 0xFF00u : 0u);  // bytes of the e4m3 pair
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int idx = threadIdx.x + kThreads * u;
    const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
    uint32_t out[2] = {0, 0};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint64_t x = f2_from_h2(w[e]);
      const float2 y = f2_unpack(div2_rn(x, nd2[e], r2[e]));
      const float2 xf = f2_unpack(x);
      // the correction's adds turn a -0 quotient into +0: the sign of x is
      // put back (E4M3 encodes -0 as 0x80)
      out[e >> 1] |= (pack_e4m3x2(copysignf(y.x, xf.x), copysignf(y.y, xf.y)) & keep[e]) << ((e & 1) * 16);
    }
    if (idx / TPR < rows) dst[idx] = make_uint2(out[0], out[1]);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 4) k_quant(const QuantJobs J) {
  constexpr int TPR = D / 8;                  // uint4 per token row
  constexpr int U = 128 * TPR / kThreads;     // uint4 per thread
  constexpr int RPU = kThreads / TPR;         // rows between a thread's uint4s
  __shared__ float s_red[kThreads / 32];

  int job = blockIdx.x;
  int kind;  // 0 = Q, 1 = K, 2 = V
  if (job < J.n_q) {
    kind = 0;
  } else if (job < J.n_q + J.n_k) {
    kind = 1;
    job -= J.n_q;
  } else {
    quant_v_block<D>(J, (job - J.n_q - J.n_k) / J.nb, (job - J.n_q - J.n_k) % J.nb);
    return;
  }
  const int slab = job / J.nb, blk = job % J.nb;
  size_t srow;
  int len;
  slab_rows(J.seq, slab, kind == 0 ? J.H : J.Hkv, &srow, &len);
  const int rows = min(128, len - blk * 128);
  if (rows <= 0) return;  // a block past the end of a short sequence
  const size_t row0 = srow + static_cast<size_t>(blk) * 128;
  const uint4* src = (kind == 0 ? J.q : J.k) + row0 * TPR;
  uint2* dst = (kind == 0 ? J.q_hat : J.k_hat) + row0 * TPR;
  const int cg = threadIdx.x % TPR;  // this thread's 8 channels: cg*8 .. cg*8+7 (fixed across u)
  const int rl = threadIdx.x / TPR;  // this thread's first row

  uint4 raw[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int idx = threadIdx.x + kThreads * u;
    raw[u] = (idx / TPR < rows) ? ld_stream(src + idx) : make_uint4(0, 0, 0, 0);
  }

  // x = fp32(q) * sm_scale or fp32(k) - mean_k.  The block absmax is taken
  // on the fp16 values (rounding is monotonic: max |fl(f s)| = fl(max |f| s)
  // and, per channel, max |fl(f - m)| = max(|fl(max f - m)|, |fl(min f - m)|)).
  float amax = 0.f;
  uint64_t m2[4];
  if (kind == 0) {
    uint32_t mag = 0;  // two fp16 magnitudes (rows past the end are +0)
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) mag = __vmaxu2(mag, w[e] & 0x7FFF7FFFu);
    }
    const uint32_t mx = max(mag & 0xFFFFu, mag >> 16);
    amax = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(mx))), fabsf(J.sm_scale));
  } else {
    const float* mk = J.mean_k + static_cast<size_t>(slab) * D + cg * 8;
#pragma unroll
    for (int e = 0; e < 4; ++e) m2[e] = f2_pack(mk[2 * e], mk[2 * e + 1]);
    if (rl < rows) {  // u = 0 is this thread's first row; later ones may be past the end
      __half2 cmax[4], cmin[4];
      {
        const uint32_t w[4] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) cmax[e] = cmin[e] = *reinterpret_cast<const __half2*>(&w[e]);
      }
#pragma unroll
      for (int u = 1; u < U; ++u) {
        if (rl + u * RPU < rows) {
          const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __half2 v = *reinterpret_cast<const __half2*>(&w[e]);
            cmax[e] = __hmax2(cmax[e], v);
            cmin[e] = __hmin2(cmin[e], v);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 a = f2_unpack(f2_sub(f2_from_h2(*reinterpret_cast<const uint32_t*>(&cmax[e])), m2[e]));
        const float2 b = f2_unpack(f2_sub(f2_from_h2(*reinterpret_cast<const uint32_t*>(&cmin[e])), m2[e]));
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b.x), fabsf(b.y))));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = s_red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) amax = fmaxf(amax, s_red[i]);

  const float delta = __fdiv_rn(amax, 127.f);
  if (threadIdx.x == 0) (kind == 0 ? J.delta_q : J.delta_k)[static_cast<size_t>(slab) * J.nb + blk] = delta;
  const float r = delta != 0.f ? __frcp_rn(delta) : 0.f;
  const uint64_t r2 = f2_pack(r, r), nd2 = f2_pack(-delta, -delta), s2 = f2_pack(J.sm_scale, J.sm_scale);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int idx = threadIdx.x + kThreads * u;
    if (idx / TPR >= rows) continue;
    const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
    uint64_t x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = kind == 0 ? f2_mul(f2_from_h2(w[e]), s2) : f2_sub(f2_from_h2(w[e]), m2[e]);
    uint2 out = make_uint2(0u, 0u);
    if (delta != 0.f) out = make_uint2(codes4(x[0], x[1], nd2, r2), codes4(x[2], x[3], nd2, r2));
    dst[idx] = out;
  }
}

// Q and K blocks with rotary embedding: one CTA per (128-token block, G
// consecutive heads of one batch entry, Q or K); jobs [0, n_q) are Q
// groups, [n_q, n_q + n_k) K groups, then n_v V blocks (one head each, no
// rotation, as in k_quant).  The block's cos / sin rows are staged
// once in shared memory, then each head's block is rotated and quantized
// with the values of k_quant: x = fp32(q) * sm_scale or fp32(k) - mean_k,
// delta = RN(absmax / 127), codes RN(x / delta).  A thread holds channel
// groups j and j + TP (both halves of its rotation pairs) of rows
// rl + u * RPP.  The block absmax is taken on the rotated fp16 values: fp32
// rounding is monotonic, so max |fl(f s)| = fl(max |f| * s) and, per
// channel, max |fl(f - m)| = max(|fl(max f - m)|, |fl(min f - m)|).
template <int D>
constexpr int rope_tab_bytes() { return 128 * D * 4; }  // cos and sin, D/2 each, of 128 tokens

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 3) k_quant_rope(const QuantJobs J) {
  constexpr int TPR = D / 8, TP = TPR / 2, H2 = D / 2;
  constexpr int RPP = kThreads / TP;  // rows per pass
  constexpr int R = 128 / RPP;        // rows per thread
  // [token][quarter][j] float4; quarters: cos of frequencies 8j..8j+3,
  // cos of 8j+4..8j+7, then the same of sin (lanes j read adjacent 16 bytes)
  extern __shared__ float4 s_tab[];
  __shared__ float s_red[2][kThreads / 32];

  int job = blockIdx.x;
  if (job >= J.n_q + J.n_k) {  // V: no rotation
    job -= J.n_q + J.n_k;
    quant_v_block<D>(J, job / J.nb, job % J.nb);
    return;
  }
  const int kind = job < J.n_q ? 0 : 1;
  if (kind == 1) job -= J.n_q;
  const int Hs = kind == 0 ? J.H : J.Hkv;
  const int z0 = (job / J.nb) * G, blk = job % J.nb;
  size_t srow;
  int len;
  slab_rows(J.seq, z0, Hs, &srow, &len);  // the same tokens for all G heads
  const int rows = min(128, len - blk * 128);
  if (rows <= 0) return;  // a block past the end of a short sequence
  // head z0 + h starts T rows after head z0 + h - 1 (both layouts)
  const size_t row_b = srow + static_cast<size_t>(blk) * 128;
  const uint4* src0 = (kind == 0 ? J.q : J.k) + row_b * TPR;
  uint2* dst0 = (kind == 0 ? J.q_hat : J.k_hat) + row_b * TPR;
  const size_t hstride = static_cast<size_t>(J.seq.T) * TPR;
  float* dlt = (kind == 0 ? J.delta_q : J.delta_k) + static_cast<size_t>(z0) * J.nb + blk;
  const int j = threadIdx.x % TP, rl = threadIdx.x / TP;

  // FULL: all 128 rows present (no per-row predicates)
  auto run = [&](auto full_tag) {
    constexpr bool FULL = decltype(full_tag)::value;
    uint4 lo[R], hi[R];
    auto load_block = [&](int h) {
      const uint4* src = src0 + h * hstride;
#pragma unroll
      for (int u = 0; u < R; ++u) {
        const int row = rl + u * RPP;
        const bool in = FULL || row < rows;
        lo[u] = in ? ld_stream(src + row * TPR + j) : make_uint4(0, 0, 0, 0);
        hi[u] = in ? ld_stream(src + row * TPR + j + TP) : make_uint4(0, 0, 0, 0);
      }
    };
    load_block(0);  // in flight while the table is staged
    {
      const float* tabs[2] = {J.cos_t + static_cast<size_t>(blk) * 128 * H2,
                              J.sin_t + static_cast<size_t>(blk) * 128 * H2};
#pragma unroll 2
      for (int i = threadIdx.x; i < 2 * 128 * (H2 / 4); i += kThreads) {
        const int tab = i / (128 * (H2 / 4)), row = (i / (H2 / 4)) % 128, f4 = i % (H2 / 4);
        if (FULL || row < rows)
          s_tab[(row * 4 + tab * 2 + (f4 & 1)) * TP + (f4 >> 1)] = ld_f4(tabs[tab] + row * H2 + 4 * f4);
      }
    }
    __syncthreads();

    for (int h = 0; h < G; ++h) {
      if (h > 0) load_block(h);
#pragma unroll
      for (int u = 0; u < R; ++u) {
        const int row = rl + u * RPP;
        if (FULL || row < rows) {  // table rows past the end are not staged
          const float4* t = s_tab + row * 4 * TP + j;
          const float4 c0 = t[0], c1 = t[TP], s0 = t[2 * TP], s1 = t[3 * TP];
          rope2(lo[u].x, hi[u].x, f2_pack(c0.x, c0.y), f2_pack(s0.x, s0.y));
          rope2(lo[u].y, hi[u].y, f2_pack(c0.z, c0.w), f2_pack(s0.z, s0.w));
          rope2(lo[u].z, hi[u].z, f2_pack(c1.x, c1.y), f2_pack(s1.x, s1.y));
          rope2(lo[u].w, hi[u].w, f2_pack(c1.z, c1.w), f2_pack(s1.z, s1.w));
        }
      }
      // this thread's share of the block absmax
      float amax = 0.f;
      uint64_t m2[8];  // K: mean_k of channels 8j.. (m2[0..3]) and H2+8j.. (m2[4..7]), in pairs
      if (kind == 0) {
        uint32_t mag = 0;  // two fp16 magnitudes (rows past the end are +0)
#pragma unroll
        for (int u = 0; u < R; ++u) {
          const uint32_t w[8] = {lo[u].x, lo[u].y, lo[u].z, lo[u].w, hi[u].x, hi[u].y, hi[u].z, hi[u].w};
#pragma unroll
          for (int e = 0; e < 8; ++e) mag = __vmaxu2(mag, w[e] & 0x7FFF7FFFu);
        }
        const uint32_t mx = max(mag & 0xFFFFu, mag >> 16);
        amax = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(mx))), fabsf(J.sm_scale));
      } else {
        const float* mk = J.mean_k + static_cast<size_t>(z0 + h) * D;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          m2[e] = f2_pack(mk[8 * j + 2 * e], mk[8 * j + 2 * e + 1]);
          m2[4 + e] = f2_pack(mk[H2 + 8 * j + 2 * e], mk[H2 + 8 * j + 2 * e + 1]);
        }
        if (FULL || rl < rows) {  // row rl (u = 0) is this thread's first; others may be past the end
          __half2 cmax[8], cmin[8];
          {
            const uint32_t w[8] = {lo[0].x, lo[0].y, lo[0].z, lo[0].w, hi[0].x, hi[0].y, hi[0].z, hi[0].w};
#pragma unroll
            for (int e = 0; e < 8; ++e) cmax[e] = cmin[e] = *reinterpret_cast<const __half2*>(&w[e]);
          }
#pragma unroll
          for (int u = 1; u < R; ++u) {
            if (FULL || rl + u * RPP < rows) {
              const uint32_t w[8] = {lo[u].x, lo[u].y, lo[u].z, lo[u].w, hi[u].x, hi[u].y, hi[u].z, hi[u].w};
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const __half2 v = *reinterpret_cast<const __half2*>(&w[e]);
                cmax[e] = __hmax2(cmax[e], v);
                cmin[e] = __hmin2(cmin[e], v);
              }
            }
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 a = f2_unpack(f2_sub(f2_from_h2(*reinterpret_cast<const uint32_t*>(&cmax[e])), m2[e]));
            const float2 b = f2_unpack(f2_sub(f2_from_h2(*reinterpret_cast<const uint32_t*>(&cmin[e])), m2[e]));
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b.x), fabsf(b.y))));
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      // one barrier per head: s_red alternates, and a warp writes slot h & 1
      // again (head h + 2) only after every warp passed head h + 1's barrier,
      // i.e. after it read head h's slot
      if ((threadIdx.x & 31) == 0) s_red[h & 1][threadIdx.x >> 5] = amax;
      __syncthreads();
      amax = s_red[h & 1][0];
#pragma unroll
      for (int i = 1; i < kThreads / 32; ++i) amax = fmaxf(amax, s_red[h & 1][i]);
      const float delta = __fdiv_rn(amax, 127.f);
      if (threadIdx.x == 0) dlt[static_cast<size_t>(h) * J.nb] = delta;
      const float r = delta != 0.f ? __frcp_rn(delta) : 0.f;
      const uint64_t r2 = f2_pack(r, r), nd2 = f2_pack(-delta, -delta), s2 = f2_pack(J.sm_scale, J.sm_scale);
      uint2* dst = dst0 + h * hstride;
#pragma unroll
      for (int u = 0; u < R; ++u) {
        const int row = rl + u * RPP;
        if (!FULL && row >= rows) continue;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint4 v = half ? hi[u] : lo[u];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint64_t x[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            x[e] = kind == 0 ? f2_mul(f2_from_h2(w[e]), s2) : f2_sub(f2_from_h2(w[e]), m2[half * 4 + e]);
          uint2 out = make_uint2(0u, 0u);
          if (delta != 0.f) out = make_uint2(codes4(x[0], x[1], nd2, r2), codes4(x[2], x[3], nd2, r2));
          dst[row * TPR + j + half * TP] = out;
        }
      }
    }
  };
  if (rows == 128) run(std::true_type());
  else run(std::false_type());
}

// ---------------------------------------------------------------- launchers
size_t stat_chunks(int N) { return static_cast<size_t>((N + kStatRows - 1) / kStatRows); }

// The fixed layout is the packed one's special case of equal lengths
// (offsets computed instead of read): N rows per slab.
static SeqLayout fixed_or(SeqLayout seq, int N) {
  if (seq.cu == nullptr) {
    seq.T = N;
    seq.max_len = N;
  }
  return seq;
}

cudaError_t launch_colstats(const void* k, const void* v, int slabs, int N, int D,
                            long long* ksum, uint32_t* vmax, cudaStream_t st, const float* cos_t,
                            const float* sin_t, SeqLayout seq, int Hkv) {
  seq = fixed_or(seq, N);
  const int nchunk = static_cast<int>(stat_chunks(seq.max_len));
  if (nchunk == 0 || slabs == 0) return cudaSuccess;
  const uint4* k4 = static_cast<const uint4*>(k);
  const uint4* v4 = static_cast<const uint4*>(v);
  if (cos_t != nullptr && k != nullptr) {
    // rotated K sums, with the V maxima in the same pass; without V, K of
    // two heads per CTA share the table loads
    if (v4 != nullptr) {
      const dim3 grid(nchunk, slabs);
      if (D == 128) k_colstats_rope<128, 1, 2><<<grid, kThreads, 0, st>>>(k4, v4, seq, Hkv, nchunk, ksum, vmax, cos_t, sin_t);
      else k_colstats_rope<64, 1, 2><<<grid, kThreads, 0, st>>>(k4, v4, seq, Hkv, nchunk, ksum, vmax, cos_t, sin_t);
    } else {
      const int G = Hkv % 2 == 0 ? 2 : 1;
      const dim3 grid(nchunk, slabs / G);
      if (D == 128) {
        if (G == 2) k_colstats_rope<128, 2, 1><<<grid, kThreads, 0, st>>>(k4, nullptr, seq, Hkv, nchunk, ksum, nullptr, cos_t, sin_t);
        else k_colstats_rope<128, 1, 2><<<grid, kThreads, 0, st>>>(k4, nullptr, seq, Hkv, nchunk, ksum, nullptr, cos_t, sin_t);
      } else {
        if (G == 2) k_colstats_rope<64, 2, 1><<<grid, kThreads, 0, st>>>(k4, nullptr, seq, Hkv, nchunk, ksum, nullptr, cos_t, sin_t);
        else k_colstats_rope<64, 1, 2><<<grid, kThreads, 0, st>>>(k4, nullptr, seq, Hkv, nchunk, ksum, nullptr, cos_t, sin_t);
      }
    }
    k4 = nullptr;
    v4 = nullptr;
    ksum = nullptr;
  }
  if (k4 != nullptr || v4 != nullptr) {
    const dim3 grid(nchunk, slabs);
    if (D == 128) k_colstats<128><<<grid, kThreads, 0, st>>>(k4, v4, seq, Hkv, nchunk, ksum, vmax);
    else k_colstats<64><<<grid, kThreads, 0, st>>>(k4, v4, seq, Hkv, nchunk, ksum, vmax);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) set_error_detail("column statistics kernel launch", e);
  return e;
}

cudaError_t launch_finalize(const long long* ksum, const uint32_t* vmax, int slabs, int N, int D,
                            float v_r, float* mean_k, float* delta_v, cudaStream_t st, SeqLayout seq,
                            int Hkv) {
  seq = fixed_or(seq, N);
  const int nchunk = static_cast<int>(stat_chunks(seq.max_len));
  if (slabs == 0) return cudaSuccess;
  k_finalize<<<dim3(slabs, D / 32), kFinWarps * 32, 0, st>>>(ksum, vmax, nchunk, D, seq, Hkv, v_r, mean_k, delta_v);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) set_error_detail("finalize kernel launch", e);
  return e;
}

// Opt-in to the rotary table's dynamic shared memory, once per device and
// instantiation (the attribute is per device).
template <int D, int G>
static cudaError_t quant_rope_attr() {
  constexpr int kMaxDev = 64;
  static std::atomic<bool> done[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(k_quant_rope<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, rope_tab_bytes<D>());
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

template <int D, int G>
static cudaError_t launch_quant_rope(const QuantJobs& J, int total, cudaStream_t st) {
  cudaError_t e = quant_rope_attr<D, G>();
  if (e != cudaSuccess) {
    set_error_detail("cudaFuncSetAttribute(rotary quantization)", e, rope_tab_bytes<D>());
    return e;
  }
  k_quant_rope<D, G><<<total, kThreads, rope_tab_bytes<D>(), st>>>(J);
  return cudaSuccess;
}

cudaError_t launch_quant(const QuantArgs& a, cudaStream_t st) {
  QuantJobs J;
  J.q = static_cast<const uint4*>(a.q);
  J.k = static_cast<const uint4*>(a.k);
  J.v = static_cast<const uint4*>(a.v);
  J.q_hat = reinterpret_cast<uint2*>(a.q_hat);
  J.k_hat = reinterpret_cast<uint2*>(a.k_hat);
  J.v_hat = reinterpret_cast<uint2*>(a.v_hat);
  J.delta_q = a.delta_q;
  J.delta_k = a.delta_k;
  J.mean_k = a.mean_k;
  J.delta_v = a.delta_v;
  J.sm_scale = a.sm_scale;
  J.cos_t = a.cos_t;
  J.sin_t = a.sin_t;
  J.seq = fixed_or(a.seq, a.N);
  J.H = a.H;
  J.Hkv = a.H_kv;
  J.nb = (J.seq.max_len + 127) / 128;
  J.n_q = a.q ? a.B * a.H * J.nb : 0;
  J.n_k = a.k ? a.B * a.H_kv * J.nb : 0;
  J.n_v = a.v ? a.B * a.H_kv * J.nb : 0;
  if (J.n_q + J.n_k + J.n_v == 0) return cudaSuccess;
  if (a.cos_t != nullptr && J.n_q + J.n_k > 0) {
    // Q and K in head groups with the rotary table, V blocks after them
    const int G = std::min(rope_group(a.H), rope_group(a.H_kv));
    QuantJobs R = J;
    R.n_q = J.n_q / G;
    R.n_k = J.n_k / G;
    const int total = R.n_q + R.n_k + R.n_v;
    cudaError_t e;
    if (a.d == 128) {
      e = G == 4 ? launch_quant_rope<128, 4>(R, total, st)
                 : G == 2 ? launch_quant_rope<128, 2>(R, total, st) : launch_quant_rope<128, 1>(R, total, st);
    } else {
      e = G == 4 ? launch_quant_rope<64, 4>(R, total, st)
                 : G == 2 ? launch_quant_rope<64, 2>(R, total, st) : launch_quant_rope<64, 1>(R, total, st);
    }
    if (e != cudaSuccess) return e;
    J.n_q = 0;
    J.n_k = 0;
    J.n_v = 0;
  }
  const int total = J.n_q + J.n_k + J.n_v;
  if (total > 0) {
    if (a.d == 128) k_quant<128><<<total, kThreads, 0, st>>>(J);
    else k_quant<64><<<total, kThreads, 0, st>>>(J);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) set_error_detail("quantization kernel launch", e);
  return e;
}

}  // namespace sage
