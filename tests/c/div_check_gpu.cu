// Device check of the pre-pass's paired division (csrc/quant_pair.cuh)
// against IEEE fp32 division (__fdiv_rn), bit for bit, over the inputs the
// quantizers can see:
//   int8 quantizers: delta = RN(absmax / 127) for every positive finite fp16
//     absmax, every finite fp16 x with |x| <= absmax: the quotient (up to the
//     sign of a zero) and the int8 code of codes4;
//   E4M3 quantizer: delta = RN(colmax / V_r), V_r in {448, 9}, every fp16 x
//     with |x| <= colmax: the quotient with the sign of x restored;
//   divisors with an all-ones significand and powers of two, 2^-40 .. 2^8,
//     with every fp16 x within 127 delta.
// Prints "ok <count>" or the first mismatches and exits non-zero.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <cuda_fp16.h>

#include "quant_pair.cuh"

using namespace sage;

struct Counts {
  unsigned long long checked, bad;
  float ex[4][3];  // first mismatches: x, delta, quotient
};

__device__ __forceinline__ float half_bits(uint32_t h) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

// kind 0: int8 (quotient up to the sign of zero, and the code); kind 1:
// E4M3 (quotient with the sign of x)
__global__ void check(int kind, int ndiv, const float* divs, const float* lims, Counts* out) {
  const int di = blockIdx.x;
  if (di >= ndiv) return;
  const float d = divs[di], lim = lims[di];
  const float r = __frcp_rn(d);
  const uint64_t r2 = f2_pack(r, r), nd2 = f2_pack(-d, -d);
  unsigned long long checked = 0;
  // x codes in groups of four consecutive fp16 bit patterns
  for (uint32_t h0 = threadIdx.x * 4; h0 < 65536u; h0 += blockDim.x * 4) {
    float x[4];
    bool use[4];
    for (int e = 0; e < 4; ++e) {
      const uint32_t h = h0 + e;
      x[e] = half_bits(h);
      use[e] = ((h >> 10) & 31u) != 31u && fabsf(x[e]) <= lim;
      if (!use[e]) x[e] = 0.f;
    }
    const uint64_t x01 = f2_pack(x[0], x[1]), x23 = f2_pack(x[2], x[3]);
    const float2 y01 = f2_unpack(div2_rn(x01, nd2, r2)), y23 = f2_unpack(div2_rn(x23, nd2, r2));
    const float y[4] = {y01.x, y01.y, y23.x, y23.y};
    const uint32_t codes = codes4(x01, x23, nd2, r2);
    for (int e = 0; e < 4; ++e) {
      if (!use[e]) continue;
      ++checked;
      const float want = __fdiv_rn(x[e], d);
      bool ok;
      if (kind == 0) {
        const uint32_t code = __float_as_uint(__fadd_rn(want, 12582912.f)) & 0xFFu;
        ok = (y[e] == want) && (((codes >> (8 * e)) & 0xFFu) == code);
      } else {
        ok = __float_as_uint(copysignf(y[e], x[e])) == __float_as_uint(want);
      }
      if (!ok) {
        const unsigned long long k = atomicAdd(&out->bad, 1ull);
        if (k < 4) {
          out->ex[k][0] = x[e];
          out->ex[k][1] = d;
          out->ex[k][2] = y[e];
        }
      }
    }
  }
  atomicAdd(&out->checked, checked);
}

static float host_half(uint32_t h) {
  const uint32_t s = (h >> 15) & 1u, e = (h >> 10) & 31u, m = h & 1023u;
  float v = e == 0 ? ldexpf(static_cast<float>(m), -24) : ldexpf(static_cast<float>(m | 1024u), static_cast<int>(e) - 25);
  return s ? -v : v;
}

// delta = RN(a / vr) computed on the device (IEEE division)
__global__ void make_deltas(int n, const float* a, float vr, float* d) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) d[i] = __fdiv_rn(a[i], vr);
}

static int run(int kind, int n, const float* h_div, const float* h_lim, bool divs_are_maxima, float vr,
               Counts* d_out, unsigned long long* total) {
  float *d_div, *d_lim, *d_a;
  if (cudaMalloc(&d_div, n * 4) || cudaMalloc(&d_lim, n * 4) || cudaMalloc(&d_a, n * 4)) return 2;
  cudaMemcpy(d_lim, h_lim, n * 4, cudaMemcpyHostToDevice);
  if (divs_are_maxima) {
    cudaMemcpy(d_a, h_div, n * 4, cudaMemcpyHostToDevice);
    make_deltas<<<(n + 255) / 256, 256>>>(n, d_a, vr, d_div);
  } else {
    cudaMemcpy(d_div, h_div, n * 4, cudaMemcpyHostToDevice);
  }
  cudaMemset(d_out, 0, sizeof(Counts));
  check<<<n, 256>>>(kind, n, d_div, d_lim, d_out);
  Counts h;
  if (cudaMemcpy(&h, d_out, sizeof(Counts), cudaMemcpyDeviceToHost) != cudaSuccess) return 2;
  cudaFree(d_div);
  cudaFree(d_lim);
  cudaFree(d_a);
  *total += h.checked;
  if (h.bad) {
    printf("kind %d: %llu mismatches of %llu\n", kind, h.bad, h.checked);
    for (unsigned long long k = 0; k < h.bad && k < 4; ++k)
      printf("  x=%a d=%a got=%a\n", h.ex[k][0], h.ex[k][1], h.ex[k][2]);
    return 1;
  }
  return 0;
}

int main() {
  Counts* d_out;
  if (cudaMalloc(&d_out, sizeof(Counts)) != cudaSuccess) {
    printf("no device\n");
    return 2;
  }
  unsigned long long total = 0;
  int rc = 0;
  // every positive finite fp16 maximum: int8 (/127) and E4M3 (/448, /9)
  const int nmax = 0x7C00 - 1;
  float* amax = new float[nmax];
  for (int i = 0; i < nmax; ++i) amax[i] = host_half(static_cast<uint32_t>(i + 1));
  rc |= run(0, nmax, amax, amax, true, 127.f, d_out, &total);
  rc |= run(1, nmax, amax, amax, true, 448.f, d_out, &total);
  rc |= run(1, nmax, amax, amax, true, 9.f, d_out, &total);
  // all-ones significands and powers of two, x within 127 delta
  float divs[2 * 49], lims[2 * 49];
  int n = 0;
  for (int e = -40; e <= 8; ++e) {
    uint32_t ones = 0x3FFFFFFFu;
    float o;
    memcpy(&o, &ones, 4);
    divs[n] = ldexpf(o, e);
    lims[n] = 127.f * divs[n];
    ++n;
    divs[n] = ldexpf(1.f, e);
    lims[n] = 127.f * divs[n];
    ++n;
  }
  rc |= run(0, n, divs, lims, false, 0.f, d_out, &total);
  rc |= run(1, n, divs, lims, false, 0.f, d_out, &total);
  delete[] amax;
  if (rc) {
    printf("FAIL\n");
    return rc;
  }
  printf("ok %llu\n", total);
  return 0;
}
