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
//                exact fixed-point sums of K (units of 2^-24, int64) and the
//                max |V| as fp16 magnitude bits.
//   k_finalize : per (slab, channel): mean_k = fp32(fp64(sum) * 2^-24 / N),
//                delta_v = fp32(colmax) / v_r.
//   k_quant    : one CTA per 128-token block of one head, for Q, K and V:
//                block absmax -> delta -> codes.
// Every value is bit-identical to the definition whatever the grid, because
// the reductions are exact (integer sums, max) and each element's
// arithmetic is a fixed sequence of correctly rounded fp32 operations.
#include <cuda_fp16.h>
#include <stdint.h>

#include "sage_internal.h"

namespace sage {

constexpr int kStatRows = 256;  // tokens per statistics chunk
constexpr int kThreads = 256;

// fp16 bits -> exact integer value of the fp16 number times 2^24.
__device__ __forceinline__ long long fp16_fixed24(uint32_t h) {
  const uint32_t e = (h >> 10) & 31u;
  const uint32_t m = h & 1023u;
  const long long mag = e ? (static_cast<long long>(m | 1024u) << (e - 1)) : static_cast<long long>(m);
  return (h & 0x8000u) ? -mag : mag;
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <int D>
__global__ void __launch_bounds__(kThreads) k_colstats(const uint4* __restrict__ k,
                                                       const uint4* __restrict__ v, int N,
                                                       int nchunk, long long* __restrict__ ksum,
                                                       uint32_t* __restrict__ vmax) {
  constexpr int TPR = D / 8;             // threads per row: one uint4 (8 halves) each
  constexpr int RPI = kThreads / TPR;    // rows per iteration
  const int chunk = blockIdx.x, slab = blockIdx.y;
  const int cg = threadIdx.x % TPR, rl = threadIdx.x / TPR;
  const int r0 = chunk * kStatRows, r1 = min(N, r0 + kStatRows);
  const size_t base = static_cast<size_t>(slab) * N * TPR + cg;

  long long acc[8];
  uint32_t vm[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) { acc[e] = 0; vm[e] = 0; }

  for (int r = r0 + rl; r < r1; r += RPI) {
    if (k != nullptr) {
      const uint4 x = ld_stream(k + base + static_cast<size_t>(r) * TPR);
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += fp16_fixed24(w[e] & 0xFFFFu);
        acc[2 * e + 1] += fp16_fixed24(w[e] >> 16);
      }
    }
    if (v != nullptr) {
      const uint4 y = ld_stream(v + base + static_cast<size_t>(r) * TPR);
      const uint32_t w[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        vm[2 * e] = max(vm[2 * e], w[e] & 0x7FFFu);          // |fp16| ordered as integer
        vm[2 * e + 1] = max(vm[2 * e + 1], (w[e] >> 16) & 0x7FFFu);
      }
    }
  }

  __shared__ long long s_sum[RPI][D];
  __shared__ uint32_t s_max[RPI][D];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    s_sum[rl][cg * 8 + e] = acc[e];
    s_max[rl][cg * 8 + e] = vm[e];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    long long s = 0;
    uint32_t mx = 0;
#pragma unroll 4
    for (int i = 0; i < RPI; ++i) {
      s += s_sum[i][c];
      mx = max(mx, s_max[i][c]);
    }
    const size_t o = (static_cast<size_t>(slab) * nchunk + chunk) * D + c;
    if (k != nullptr) ksum[o] = s;
    if (v != nullptr) vmax[o] = mx;
  }
}

// One thread per (slab, channel).
__global__ void k_finalize(const long long* __restrict__ ksum, const uint32_t* __restrict__ vmax,
                           int nchunk, int D, int N, float v_r, float* __restrict__ mean_k,
                           float* __restrict__ delta_v) {
  const int slab = blockIdx.x, c = threadIdx.x;
  const size_t o = static_cast<size_t>(slab) * nchunk * D + c;
  if (ksum != nullptr) {
    long long s = 0;
    for (int i = 0; i < nchunk; ++i) s += ksum[o + static_cast<size_t>(i) * D];
    const double sd = __dmul_rn(__ll2double_rn(s), 0x1p-24);
    mean_k[static_cast<size_t>(slab) * D + c] = __double2float_rn(__ddiv_rn(sd, static_cast<double>(N)));
  }
  if (vmax != nullptr) {
    uint32_t m = 0;
    for (int i = 0; i < nchunk; ++i) m = max(m, vmax[o + static_cast<size_t>(i) * D]);
    const float cm = __half2float(__ushort_as_half(static_cast<unsigned short>(m)));
    delta_v[static_cast<size_t>(slab) * D + c] = __fdiv_rn(cm, v_r);
  }
}

// Correctly rounded x / d given r = RN(1/d) (Markstein's correction step,
// P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990): q = RN(x*r) is
// within one ulp of x/d, the remainder x - q*d is exact in one fma, and
// RN(q + rem*r) is the correctly rounded quotient.  Valid away from
// overflow/underflow, which the quantizer's ranges never reach.  The
// correction's additions turn a -0 quotient into +0; with d > 0 the quotient
// carries the sign of x, which copysign restores (E4M3 encodes -0 as 0x80).
__device__ __forceinline__ float div_rn_by(float x, float d, float r) {
  const float q = __fmul_rn(x, r);
  const float rem = __fmaf_rn(-q, d, x);
  return copysignf(__fmaf_rn(rem, r, q), x);
}

// Round-half-even of |y| <= 127 to an int8 code: adding 1.5*2^23 leaves the
// rounded integer in the low mantissa bits (the fp32 add rounds to nearest
// even at unit spacing), whose low byte is the two's-complement code.
__device__ __forceinline__ uint32_t rne_code8(float y) {
  y = fminf(fmaxf(y, -127.f), 127.f);
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
  int N, nb;
  int n_q, n_k, n_v;    // number of (slab, block) jobs of each kind
};

template <int D>
__global__ void __launch_bounds__(kThreads) k_quant(const QuantJobs J) {
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
  const int rows = min(128, J.N - blk * 128);
  const size_t row0 = static_cast<size_t>(slab) * J.N + static_cast<size_t>(blk) * 128;
  const uint4* src = (kind == 0 ? J.q : kind == 1 ? J.k : J.v) + row0 * TPR;
  uint2* dst = (kind == 0 ? J.q_hat : kind == 1 ? J.k_hat : J.v_hat) + row0 * TPR;
  const int cg = threadIdx.x % TPR;  // this thread's 8 channels: cg*8 .. cg*8+7 (fixed across u)

  uint4 raw[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int idx = threadIdx.x + kThreads * u;
    raw[u] = (idx / TPR < rows) ? ld_stream(src + idx) : make_uint4(0, 0, 0, 0);
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

  float x[U][8];
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
      if (kind == 0) {
        x[u][2 * e] = __fmul_rn(f.x, J.sm_scale);
        x[u][2 * e + 1] = __fmul_rn(f.y, J.sm_scale);
      } else {
        x[u][2 * e] = __fsub_rn(f.x, sub[2 * e]);
        x[u][2 * e + 1] = __fsub_rn(f.y, sub[2 * e + 1]);
      }
    }
    const int idx = threadIdx.x + kThreads * u;
    if (idx / TPR < rows) {
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[u][e]));
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
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t b[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        b[e] = delta != 0.f ? rne_code8(div_rn_by(x[u][4 * h + e], delta, r)) : 0u;
      out[h] = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    }
    if (idx / TPR < rows) dst[idx] = make_uint2(out[0], out[1]);
  }
}

// ---------------------------------------------------------------- launchers
size_t stat_chunks(int N) { return static_cast<size_t>((N + kStatRows - 1) / kStatRows); }

cudaError_t launch_colstats(const void* k, const void* v, int slabs, int N, int D,
                            long long* ksum, uint32_t* vmax, cudaStream_t st) {
  const int nchunk = static_cast<int>(stat_chunks(N));
  dim3 grid(nchunk, slabs);
  if (D == 128)
    k_colstats<128><<<grid, kThreads, 0, st>>>(static_cast<const uint4*>(k),
                                               static_cast<const uint4*>(v), N, nchunk, ksum, vmax);
  else
    k_colstats<64><<<grid, kThreads, 0, st>>>(static_cast<const uint4*>(k),
                                              static_cast<const uint4*>(v), N, nchunk, ksum, vmax);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) set_error_detail("column statistics kernel launch", e);
  return e;
}

cudaError_t launch_finalize(const long long* ksum, const uint32_t* vmax, int slabs, int N, int D,
                            float v_r, float* mean_k, float* delta_v, cudaStream_t st) {
  const int nchunk = static_cast<int>(stat_chunks(N));
  k_finalize<<<slabs, D, 0, st>>>(ksum, vmax, nchunk, D, N, v_r, mean_k, delta_v);
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
  J.N = a.N;
  J.nb = (a.N + 127) / 128;
  J.n_q = a.q ? a.B * a.H * J.nb : 0;
  J.n_k = a.k ? a.B * a.H_kv * J.nb : 0;
  J.n_v = a.v ? a.B * a.H_kv * J.nb : 0;
  const int total = J.n_q + J.n_k + J.n_v;
  if (total == 0) return cudaSuccess;
  if (a.d == 128)
    k_quant<128><<<total, kThreads, 0, st>>>(J);
  else
    k_quant<64><<<total, kThreads, 0, st>>>(J);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) set_error_detail("quantization kernel launch", e);
  return e;
}

}  // namespace sage
