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
// With rotary tables, k_colstats and k_quant first rotate each fp16 row of K
// (and Q) in registers ([SA1] implementation detail 1: RoPE and the
// quantization in one pass, no rotated copy in HBM).
// Every value is bit-identical to the definition whatever the grid, because
// the reductions are exact (integer sums, max) and each element's
// arithmetic is a fixed sequence of correctly rounded fp32 operations.
#include <cuda_fp16.h>
#include <stdint.h>

#include "quant_div.h"
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

// Rotary embedding of the 8 fp16 channels this thread holds at token t
// (rotate-half pairing: channel i < D/2 pairs with i + D/2).  The partner
// channels sit in lane ^ (TPR/2) of the same warp; the two partners load the
// cos and the sin of their common 8 frequencies respectively and swap them.
//   lower half: y = fl(fl(x*c) - fl(x'*s)),  upper half: y = fl(fl(x*c) + fl(x'*s)),
// rounded to fp16.  t < 0 (a row past the end) yields zeros.  Every lane of
// the warp must call this (shuffles).
template <int D>
__device__ __forceinline__ uint4 rope8(uint4 x, int t, int cg, const float* __restrict__ cosT,
                                       const float* __restrict__ sinT) {
  constexpr int TPR = D / 8, H2 = D / 2;
  const bool upper = cg >= TPR / 2;
  uint4 xp;
  xp.x = __shfl_xor_sync(0xFFFFFFFFu, x.x, TPR / 2);
  xp.y = __shfl_xor_sync(0xFFFFFFFFu, x.y, TPR / 2);
  xp.z = __shfl_xor_sync(0xFFFFFFFFu, x.z, TPR / 2);
  xp.w = __shfl_xor_sync(0xFFFFFFFFu, x.w, TPR / 2);
  const float* tab = (upper ? sinT : cosT) + static_cast<size_t>(t < 0 ? 0 : t) * H2 + (cg % (TPR / 2)) * 8;
  float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
  if (t >= 0) {
    a0 = ld_f4(tab);
    a1 = ld_f4(tab + 4);
  }
  float4 b0, b1;
  b0.x = __shfl_xor_sync(0xFFFFFFFFu, a0.x, TPR / 2);
  b0.y = __shfl_xor_sync(0xFFFFFFFFu, a0.y, TPR / 2);
  b0.z = __shfl_xor_sync(0xFFFFFFFFu, a0.z, TPR / 2);
  b0.w = __shfl_xor_sync(0xFFFFFFFFu, a0.w, TPR / 2);
  b1.x = __shfl_xor_sync(0xFFFFFFFFu, a1.x, TPR / 2);
  b1.y = __shfl_xor_sync(0xFFFFFFFFu, a1.y, TPR / 2);
  b1.z = __shfl_xor_sync(0xFFFFFFFFu, a1.z, TPR / 2);
  b1.w = __shfl_xor_sync(0xFFFFFFFFu, a1.w, TPR / 2);
  const float ta[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  const float tb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
  const uint32_t w[4] = {x.x, x.y, x.z, x.w}, wp[4] = {xp.x, xp.y, xp.z, xp.w};
  uint32_t out[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
    const float2 g = __half22float2(*reinterpret_cast<const __half2*>(&wp[e]));
    const float c0 = upper ? tb[2 * e] : ta[2 * e], s0 = upper ? ta[2 * e] : tb[2 * e];
    const float c1 = upper ? tb[2 * e + 1] : ta[2 * e + 1], s1 = upper ? ta[2 * e + 1] : tb[2 * e + 1];
    const float y0 = upper ? __fadd_rn(__fmul_rn(f.x, c0), __fmul_rn(g.x, s0))
                           : __fsub_rn(__fmul_rn(f.x, c0), __fmul_rn(g.x, s0));
    const float y1 = upper ? __fadd_rn(__fmul_rn(f.y, c1), __fmul_rn(g.y, s1))
                           : __fsub_rn(__fmul_rn(f.y, c1), __fmul_rn(g.y, s1));
    const __half2 h = __floats2half2_rn(y0, y1);
    out[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

template <int D, bool ROPE>
__global__ void __launch_bounds__(kThreads) k_colstats(const uint4* __restrict__ k,
                                                       const uint4* __restrict__ v, SeqLayout seq,
                                                       int Hkv, int nchunk, long long* __restrict__ ksum,
                                                       uint32_t* __restrict__ vmax,
                                                       const float* __restrict__ cosT,
                                                       const float* __restrict__ sinT) {
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
  // (all lanes of a warp run the same iterations: the rotary path shuffles)
  for (int r = r0 + rl, rw = r0 + (rl & ~(32 / TPR - 1)); rw < r1; r += kUnroll * RPI, rw += kUnroll * RPI) {
    uint4 xk[kUnroll], xv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int rr = r + u * RPI;
      const bool in = rr < r1;
      xk[u] = (k != nullptr && in) ? ld_stream(k + base + static_cast<size_t>(rr) * TPR) : make_uint4(0, 0, 0, 0);
      xv[u] = (v != nullptr && in) ? ld_stream(v + base + static_cast<size_t>(rr) * TPR) : make_uint4(0, 0, 0, 0);
    }
    if (ROPE && k != nullptr) {
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int rr = r + u * RPI;
        xk[u] = rope8<D>(xk[u], rr < r1 ? rr : -1, cg, cosT, sinT);
      }
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

// One CTA per (slab, 32 channels): its 8 warps reduce interleaved chunks
// (lane = channel), then warp 0 combines them.  Integer sums and maxima are
// exact, so the result does not depend on this order.
__global__ void __launch_bounds__(256) k_finalize(const long long* __restrict__ ksum,
                                                  const uint32_t* __restrict__ vmax, int nchunk_max,
                                                  int D, SeqLayout seq, int Hkv, float v_r,
                                                  float* __restrict__ mean_k, float* __restrict__ delta_v) {
  const int slab = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.y * 32 + lane;
  size_t row0;
  int N;
  slab_rows(seq, slab, Hkv, &row0, &N);
  const int nchunk = (N + kStatRows - 1) / kStatRows;  // chunks written for this slab
  __shared__ long long s_s[8][32];
  __shared__ uint32_t s_m[8][32];
  long long s = 0;
  uint32_t m = 0;
  for (int i = w; i < nchunk; i += 8) {
    const size_t o = (static_cast<size_t>(slab) * nchunk_max + i) * D + c;
    if (ksum != nullptr) s += ksum[o];
    if (vmax != nullptr) m = max(m, vmax[o]);
  }
  s_s[w][lane] = s;
  s_m[w][lane] = m;
  __syncthreads();
  if (w != 0) return;
#pragma unroll
  for (int i = 1; i < 8; ++i) {
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

// Round-half-even of y to an int8 code: adding 1.5*2^23 leaves the rounded
// integer in the low mantissa bits (the fp32 add rounds to nearest even at
// unit spacing), whose low byte is the two's-complement code.  No clamp is
// needed: |x| <= absmax and delta = RN(absmax / 127) >= absmax/127 * (1 -
// 2^-24), so |RN(x / delta)| <= 127 * (1 + 2^-22) and rounds to at most 127;
// -0 and +0 both give code 0.
__device__ __forceinline__ uint32_t rne_code8(float y) {
  return __float_as_uint(__fadd_rn(y, 12582912.f)) & 0xFFu;
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

template <int D, bool ROPE>
__global__ void __launch_bounds__(kThreads, ROPE ? 3 : 4) k_quant(const QuantJobs J) {
  constexpr int TPR = D / 8;                  // uint4 per token row
  constexpr int U = 128 * TPR / kThreads;     // uint4 per thread
  __shared__ float s_red[kThreads / 32];

  int job = blockIdx.x;
  int kind;  // 0 = Q, 1 = K, 2 = V
  if (job < J.n_q) {
    kind = 0;
  } else if (job < J.n_q + J.n_k) {
    kind = 1;
    job -= J.n_q;
  } else {
    kind = 2;
    job -= J.n_q + J.n_k;
  }
  const int slab = job / J.nb, blk = job % J.nb;
  size_t srow;
  int len;
  slab_rows(J.seq, slab, kind == 0 ? J.H : J.Hkv, &srow, &len);
  const int rows = min(128, len - blk * 128);
  if (rows <= 0) return;  // a block past the end of a short sequence
  const size_t row0 = srow + static_cast<size_t>(blk) * 128;
  const uint4* src = (kind == 0 ? J.q : kind == 1 ? J.k : J.v) + row0 * TPR;
  uint2* dst = (kind == 0 ? J.q_hat : kind == 1 ? J.k_hat : J.v_hat) + row0 * TPR;
  const int cg = threadIdx.x % TPR;  // this thread's 8 channels: cg*8 .. cg*8+7 (fixed across u)

  uint4 raw[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int idx = threadIdx.x + kThreads * u;
    raw[u] = (idx / TPR < rows) ? ld_stream(src + idx) : make_uint4(0, 0, 0, 0);
  }
  if (ROPE && kind != 2) {  // kind is uniform over the CTA
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int idx = threadIdx.x + kThreads * u;
      raw[u] = rope8<D>(raw[u], idx / TPR < rows ? blk * 128 + idx / TPR : -1, cg, J.cos_t, J.sin_t);
    }
  }

  if (kind == 2) {
    // V: per-channel scale, no block reduction.
    float dv[8], rv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      dv[e] = J.delta_v[static_cast<size_t>(slab) * D + cg * 8 + e];
      rv[e] = dv[e] != 0.f ? __frcp_rn(dv[e]) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int idx = threadIdx.x + kThreads * u;
      const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
      uint32_t out[2] = {0, 0};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __half2 h = *reinterpret_cast<const __half2*>(&w[e]);
        const float2 f = __half22float2(h);
        const float y0 = dv[2 * e] != 0.f ? div_rn_by(f.x, dv[2 * e], rv[2 * e]) : 0.f;
        const float y1 = dv[2 * e + 1] != 0.f ? div_rn_by(f.y, dv[2 * e + 1], rv[2 * e + 1]) : 0.f;
        out[e >> 1] |= pack_e4m3x2(y0, y1) << ((e & 1) * 16);
      }
      if (idx / TPR < rows) dst[idx] = make_uint2(out[0], out[1]);
    }
    return;
  }

  float sub[8];
#pragma unroll
  for (int e = 0; e < 8; ++e)
    sub[e] = (kind == 1) ? J.mean_k[static_cast<size_t>(slab) * D + cg * 8 + e] : 0.f;

  // x = fp32(q) * sm_scale or fp32(k) - mean_k, formed twice (for the block
  // max and for the codes) so that only the raw loads stay live in between
  auto xval = [&](uint32_t w, int e) -> float2 {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
    return kind == 0 ? make_float2(__fmul_rn(f.x, J.sm_scale), __fmul_rn(f.y, J.sm_scale))
                     : make_float2(__fsub_rn(f.x, sub[2 * e]), __fsub_rn(f.y, sub[2 * e + 1]));
  };
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
    const int idx = threadIdx.x + kThreads * u;
    if (idx / TPR < rows) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = xval(w[e], e);
        amax = fmaxf(amax, fmaxf(fabsf(x.x), fabsf(x.y)));
      }
    }
  }
  // block absmax
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

#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int idx = threadIdx.x + kThreads * u;
    const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float2 x0 = xval(w[2 * h], 2 * h), x1 = xval(w[2 * h + 1], 2 * h + 1);
      const float xs[4] = {x0.x, x0.y, x1.x, x1.y};
      uint32_t b[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) b[e] = delta != 0.f ? rne_code8(div_rn_nosign(xs[e], delta, r)) : 0u;
      out[h] = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    }
    if (idx / TPR < rows) dst[idx] = make_uint2(out[0], out[1]);
  }
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
  dim3 grid(nchunk, slabs);
  const uint4* k4 = static_cast<const uint4*>(k);
  const uint4* v4 = static_cast<const uint4*>(v);
  const bool rope = cos_t != nullptr && k != nullptr;
  if (D == 128) {
    if (rope) k_colstats<128, true><<<grid, kThreads, 0, st>>>(k4, v4, seq, Hkv, nchunk, ksum, vmax, cos_t, sin_t);
    else k_colstats<128, false><<<grid, kThreads, 0, st>>>(k4, v4, seq, Hkv, nchunk, ksum, vmax, nullptr, nullptr);
  } else {
    if (rope) k_colstats<64, true><<<grid, kThreads, 0, st>>>(k4, v4, seq, Hkv, nchunk, ksum, vmax, cos_t, sin_t);
    else k_colstats<64, false><<<grid, kThreads, 0, st>>>(k4, v4, seq, Hkv, nchunk, ksum, vmax, nullptr, nullptr);
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
  k_finalize<<<dim3(slabs, D / 32), 256, 0, st>>>(ksum, vmax, nchunk, D, seq, Hkv, v_r, mean_k, delta_v);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) set_error_detail("finalize kernel launch", e);
  return e;
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
  const int total = J.n_q + J.n_k + J.n_v;
  if (total == 0) return cudaSuccess;
  const bool rope = a.cos_t != nullptr;
  if (a.d == 128) {
    if (rope) k_quant<128, true><<<total, kThreads, 0, st>>>(J);
    else k_quant<128, false><<<total, kThreads, 0, st>>>(J);
  } else {
    if (rope) k_quant<64, true><<<total, kThreads, 0, st>>>(J);
    else k_quant<64, false><<<total, kThreads, 0, st>>>(J);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) set_error_detail("quantization kernel launch", e);
  return e;
}

}  // namespace sage
