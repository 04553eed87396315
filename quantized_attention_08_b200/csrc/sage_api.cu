// sage_api.cu -- the C ABI declared in include/sage.h: argument checks,
// workspace carving, stream-ordered allocation and kernel launches.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "sage.h"
#include "sage_internal.h"

namespace {

std::atomic<uint64_t> g_timeout_ns{2000000000ull};

constexpr int kMaxDevices = 64;
std::atomic<int> g_dev_ok[kMaxDevices];  // 0 unknown, 1 sm_100, -1 other

sage_status_t check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SAGE_ERR_DEVICE;
  int ok = g_dev_ok[dev].load(std::memory_order_acquire);
  if (ok == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return SAGE_ERR_CUDA;
    ok = (major == 10 && minor == 0) ? 1 : -1;
    g_dev_ok[dev].store(ok, std::memory_order_release);  // every thread computes the same value
  }
  return ok == 1 ? SAGE_OK : SAGE_ERR_DEVICE;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool a4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

sage_status_t check_sizes(int B, int H, int H_kv, int N, int d) {
  if (B < 0 || H <= 0 || H_kv <= 0 || N < 0) return SAGE_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
  if (H % H_kv != 0) return SAGE_ERR_UNSUPPORTED;
  // grid.y = B*H; TMA coordinates are 32-bit
  if (static_cast<long long>(B) * H > 65535) return SAGE_ERR_UNSUPPORTED;
  if (N > (1 << 24)) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

sage_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return SAGE_OK;
  if (e == cudaErrorMemoryAllocation) return SAGE_ERR_NO_MEMORY;
  return SAGE_ERR_CUDA;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Layout of the intermediates inside one workspace.
struct WsLayout {
  size_t q_hat, k_hat, v_hat, delta_q, delta_k, mean_k, delta_v, ksum, vmax, total;
};

// T < 0: fixed layout ([B, H, N, d]); T >= 0: packed sequences ([H, T, d],
// at most N tokens each).
WsLayout ws_layout(int B, int H, int H_kv, int N, int d, int variant, long long T = -1) {
  WsLayout L;
  const size_t nb = static_cast<size_t>((N + 127) / 128);
  const size_t nq = static_cast<size_t>(B) * H, nk = static_cast<size_t>(B) * H_kv;
  const size_t nchunk = sage::stat_chunks(N);
  // rows of q (and o) and of k (and v): B*H*N and B*H_kv*N, or H*T and H_kv*T
  const size_t rq = T < 0 ? nq * N : static_cast<size_t>(H) * T;
  const size_t rk = T < 0 ? nk * N : static_cast<size_t>(H_kv) * T;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.q_hat = take(rq * d);
  L.k_hat = take(rk * d);
  const bool v8 = variant != SAGE_VARIANT_B;
  L.v_hat = take(v8 ? rk * d : 0);
  L.delta_q = take(nq * nb * 4);
  L.delta_k = take(nk * nb * 4);
  L.mean_k = take(nk * d * 4);
  L.delta_v = take(v8 ? nk * d * 4 : 0);
  L.ksum = take(nk * nchunk * d * 8);
  L.vmax = take(v8 ? nk * nchunk * d * 4 : 0);
  L.total = off;
  return L;
}

// Pre-pass for Q, K and (when v != nullptr) V with caller-provided scratch.
cudaError_t run_prepass(const void* q, const void* k, const void* v, int B, int H, int H_kv, int N,
                        int d, float sm_scale, float v_r, int8_t* q_hat, int8_t* k_hat,
                        uint8_t* v_hat, float* delta_q, float* delta_k, float* mean_k,
                        float* delta_v, long long* ksum, uint32_t* vmax, cudaStream_t st,
                        const float* cos_t = nullptr, const float* sin_t = nullptr,
                        sage::SeqLayout seq = sage::SeqLayout()) {
  const int slabs = B * H_kv;
  cudaError_t e = sage::launch_colstats(k, v, slabs, N, d, ksum, v ? vmax : nullptr, st, cos_t, sin_t, seq, H_kv);
  if (e == cudaSuccess)
    e = sage::launch_finalize(ksum, v ? vmax : nullptr, slabs, N, d, v_r, mean_k, delta_v, st, seq, H_kv);
  if (e == cudaSuccess) {
    sage::QuantArgs qa;
    qa.q = q;
    qa.k = k;
    qa.v = v;
    qa.q_hat = q_hat;
    qa.k_hat = k_hat;
    qa.v_hat = v_hat;
    qa.delta_q = delta_q;
    qa.delta_k = delta_k;
    qa.mean_k = mean_k;
    qa.delta_v = delta_v;
    qa.sm_scale = sm_scale;
    qa.B = B;
    qa.H = H;
    qa.H_kv = H_kv;
    qa.N = N;
    qa.d = d;
    qa.cos_t = cos_t;
    qa.sin_t = sin_t;
    qa.seq = seq;
    e = sage::launch_quant(qa, st);
  }
  return e;
}

// The whole pass with intermediates carved from `ws` (L.total bytes).
sage_status_t run_forward(const void* q, const void* k, const void* v, void* o, int B, int H,
                          int H_kv, int N, int d, int causal, float sm_scale, int variant,
                          uint8_t* ws, const WsLayout& L, cudaStream_t st,
                          sage::SeqLayout seq = sage::SeqLayout()) {
  const bool v8 = variant != SAGE_VARIANT_B;
  const bool r56 = variant == SAGE_VARIANT_8P8_R56;
  int8_t* q_hat = reinterpret_cast<int8_t*>(ws + L.q_hat);
  int8_t* k_hat = reinterpret_cast<int8_t*>(ws + L.k_hat);
  uint8_t* v_hat = v8 ? ws + L.v_hat : nullptr;
  float* delta_q = reinterpret_cast<float*>(ws + L.delta_q);
  float* delta_k = reinterpret_cast<float*>(ws + L.delta_k);
  float* mean_k = reinterpret_cast<float*>(ws + L.mean_k);
  float* delta_v = v8 ? reinterpret_cast<float*>(ws + L.delta_v) : nullptr;
  long long* ksum = reinterpret_cast<long long*>(ws + L.ksum);
  uint32_t* vmax = v8 ? reinterpret_cast<uint32_t*>(ws + L.vmax) : nullptr;

  cudaError_t e = run_prepass(q, k, v8 ? v : nullptr, B, H, H_kv, N, d, sm_scale, r56 ? 9.0f : 448.0f, q_hat,
                              k_hat, v_hat, delta_q, delta_k, mean_k, delta_v, ksum, vmax, st, nullptr,
                              nullptr, seq);
  if (e == cudaSuccess) {
    sage::AttnArgs aa;
    aa.q_hat = q_hat;
    aa.k_hat = k_hat;
    aa.delta_q = delta_q;
    aa.delta_k = delta_k;
    aa.v = v8 ? static_cast<const void*>(v_hat) : v;
    aa.delta_v = delta_v;
    aa.o = o;
    aa.B = B;
    aa.H = H;
    aa.H_kv = H_kv;
    aa.N = N;
    aa.d = d;
    aa.causal = causal;
    aa.variant = v8 ? 1 : 0;
    aa.p_r = r56 ? 56.f : 448.f;
    aa.timeout_ns = g_timeout_ns.load();
    aa.cu = seq.cu;
    aa.T = seq.T;
    e = sage::launch_attention(aa, st);
  }
  return from_cuda(e);
}

sage_status_t check_fwd_args(const void* q, const void* k, const void* v, void* o, int B, int H,
                             int H_kv, int N, int d, int causal, float sm_scale, int variant) {
  sage_status_t s = check_sizes(B, H, H_kv, N, d);
  if (s != SAGE_OK) return s;
  if (variant != SAGE_VARIANT_B && variant != SAGE_VARIANT_8P8 && variant != SAGE_VARIANT_8P8_R56)
    return SAGE_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return SAGE_OK;
  if (!q || !k || !v || !o) return SAGE_ERR_INVALID_ARG;
  if (!a16(q) || !a16(k) || !a16(v) || !a16(o)) return SAGE_ERR_MISALIGNED;
  return SAGE_OK;
}

}  // namespace

// ------------------------------------------------ allocation-free pre-pass
// Scratch of sage_smooth_quant_qk_noalloc: the per-(slab, 256-token chunk,
// channel) int64 partial sums of K that the column-statistics kernel writes
// and the finalize kernel reads.  It lives in the module's static device
// memory (one copy per device, created when the module is loaded), so the
// call itself never allocates.  Every entry the finalize kernel reads is
// written earlier in the same call, so nothing here has to start at zero.
constexpr size_t kNoAllocPartials = size_t(1) << 19;  // 524,288 int64 = 4 MiB
static __device__ __align__(256) long long g_noalloc_ksum[kNoAllocPartials];

namespace {

std::mutex g_noalloc_mu;
long long* g_noalloc_ptr[kMaxDevices];  // device address of g_noalloc_ksum, per device

// Set-up, once per device, with that device current.
sage_status_t noalloc_scratch(int dev, long long** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_ksum);
    if (e != cudaSuccess) {
      sage::set_error_detail("cudaGetSymbolAddress(static pre-pass scratch)", e);
      return from_cuda(e);
    }
    g_noalloc_ptr[dev] = static_cast<long long*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return SAGE_OK;
}

}  // namespace

extern "C" {

sage_status_t sage_smooth_quant_qk(const void* q, const void* k, int B, int H, int H_kv, int N,
                                   int d, float sm_scale, int8_t* q_hat, int8_t* k_hat,
                                   float* delta_q, float* delta_k, float* mean_k, void* stream) {
  sage_status_t s = check_sizes(B, H, H_kv, N, d);
  if (s != SAGE_OK) return s;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return SAGE_OK;
  if (!q || !k || !q_hat || !k_hat || !delta_q || !delta_k || !mean_k) return SAGE_ERR_INVALID_ARG;
  if (!a16(q) || !a16(k) || !a16(q_hat) || !a16(k_hat) || !a4(delta_q) || !a4(delta_k) ||
      !a4(mean_k))
    return SAGE_ERR_MISALIGNED;
  if ((s = check_device()) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int slabs = B * H_kv;
  const size_t bytes = static_cast<size_t>(slabs) * sage::stat_chunks(N) * d * 8;
  void* scratch = nullptr;
  cudaError_t e = cudaMallocAsync(&scratch, bytes, st);
  if (e != cudaSuccess) return from_cuda(e);
  long long* ksum = static_cast<long long*>(scratch);
  e = sage::launch_colstats(k, nullptr, slabs, N, d, ksum, nullptr, st);
  if (e == cudaSuccess) e = sage::launch_finalize(ksum, nullptr, slabs, N, d, 0.f, mean_k, nullptr, st);
  if (e == cudaSuccess) {
    sage::QuantArgs qa;
    std::memset(&qa, 0, sizeof(qa));
    qa.q = q;
    qa.k = k;
    qa.q_hat = q_hat;
    qa.k_hat = k_hat;
    qa.delta_q = delta_q;
    qa.delta_k = delta_k;
    qa.mean_k = mean_k;
    qa.sm_scale = sm_scale;
    qa.B = B;
    qa.H = H;
    qa.H_kv = H_kv;
    qa.N = N;
    qa.d = d;
    e = sage::launch_quant(qa, st);
  }
  cudaError_t ef = cudaFreeAsync(scratch, st);
  return from_cuda(e != cudaSuccess ? e : ef);
}

sage_status_t sage_smooth_quant_qk_noalloc(const void* q, const void* k, int B, int H, int H_kv,
                                           int N, int d, float sm_scale, int8_t* q_hat,
                                           int8_t* k_hat, float* delta_q, float* delta_k,
                                           float* mean_k, void* stream) {
  sage_status_t s = check_sizes(B, H, H_kv, N, d);
  if (s != SAGE_OK) return s;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return SAGE_OK;
  if (!q || !k || !q_hat || !k_hat || !delta_q || !delta_k || !mean_k) return SAGE_ERR_INVALID_ARG;
  if (!a16(q) || !a16(k) || !a16(q_hat) || !a16(k_hat) || !a4(delta_q) || !a4(delta_k) ||
      !a4(mean_k))
    return SAGE_ERR_MISALIGNED;
  const int slabs = B * H_kv;
  const size_t need = static_cast<size_t>(slabs) * sage::stat_chunks(N) * d;
  if (need > kNoAllocPartials) {
    sage::set_error_detail(
        "sage_smooth_quant_qk_noalloc: B*H_kv*ceil(N/256)*d partial sums exceed the static "
        "scratch of 524288 (4 MiB); use sage_smooth_quant_qk for these sizes",
        cudaErrorInvalidValue, static_cast<int>(need > 0x7FFFFFFF ? 0x7FFFFFFF : need));
    return SAGE_ERR_UNSUPPORTED;
  }
  if ((s = check_device()) != SAGE_OK) return s;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  long long* ksum = nullptr;
  if ((s = noalloc_scratch(dev, &ksum)) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = sage::launch_colstats(k, nullptr, slabs, N, d, ksum, nullptr, st);
  if (e == cudaSuccess) e = sage::launch_finalize(ksum, nullptr, slabs, N, d, 0.f, mean_k, nullptr, st);
  if (e == cudaSuccess) {
    sage::QuantArgs qa;
    std::memset(&qa, 0, sizeof(qa));
    qa.q = q;
    qa.k = k;
    qa.q_hat = q_hat;
    qa.k_hat = k_hat;
    qa.delta_q = delta_q;
    qa.delta_k = delta_k;
    qa.mean_k = mean_k;
    qa.sm_scale = sm_scale;
    qa.B = B;
    qa.H = H;
    qa.H_kv = H_kv;
    qa.N = N;
    qa.d = d;
    e = sage::launch_quant(qa, st);
  }
  return from_cuda(e);
}

sage_status_t sage_quant_v_fp8(const void* v, int B, int H_kv, int N, int d, float v_r,
                               uint8_t* v_hat, float* delta_v, void* stream) {
  sage_status_t s = check_sizes(B, H_kv, H_kv, N, d);
  if (s != SAGE_OK) return s;
  if (!(v_r > 0.f) || !(v_r <= 448.f)) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return SAGE_OK;
  if (!v || !v_hat || !delta_v) return SAGE_ERR_INVALID_ARG;
  if (!a16(v) || !a16(v_hat) || !a4(delta_v)) return SAGE_ERR_MISALIGNED;
  if ((s = check_device()) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int slabs = B * H_kv;
  const size_t bytes = static_cast<size_t>(slabs) * sage::stat_chunks(N) * d * 4;
  void* scratch = nullptr;
  cudaError_t e = cudaMallocAsync(&scratch, bytes, st);
  if (e != cudaSuccess) return from_cuda(e);
  uint32_t* vmax = static_cast<uint32_t*>(scratch);
  e = sage::launch_colstats(nullptr, v, slabs, N, d, nullptr, vmax, st);
  if (e == cudaSuccess) e = sage::launch_finalize(nullptr, vmax, slabs, N, d, v_r, nullptr, delta_v, st);
  if (e == cudaSuccess) {
    sage::QuantArgs qa;
    std::memset(&qa, 0, sizeof(qa));
    qa.v = v;
    qa.v_hat = v_hat;
    qa.delta_v = delta_v;
    qa.B = B;
    qa.H = H_kv;
    qa.H_kv = H_kv;
    qa.N = N;
    qa.d = d;
    e = sage::launch_quant(qa, st);
  }
  cudaError_t ef = cudaFreeAsync(scratch, st);
  return from_cuda(e != cudaSuccess ? e : ef);
}

sage_status_t sage_smooth_quant_qkv(const void* q, const void* k, const void* v, int B, int H,
                                    int H_kv, int N, int d, float sm_scale, float v_r,
                                    int8_t* q_hat, int8_t* k_hat, uint8_t* v_hat, float* delta_q,
                                    float* delta_k, float* mean_k, float* delta_v, void* stream) {
  sage_status_t s = check_sizes(B, H, H_kv, N, d);
  if (s != SAGE_OK) return s;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  const bool hv = v != nullptr;
  if (hv && (!(v_r > 0.f) || !(v_r <= 448.f))) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return SAGE_OK;
  if (!q || !k || !q_hat || !k_hat || !delta_q || !delta_k || !mean_k) return SAGE_ERR_INVALID_ARG;
  if (hv != (v_hat != nullptr) || hv != (delta_v != nullptr)) return SAGE_ERR_INVALID_ARG;
  if (!a16(q) || !a16(k) || !a16(q_hat) || !a16(k_hat) || !a4(delta_q) || !a4(delta_k) ||
      !a4(mean_k) || (hv && (!a16(v) || !a16(v_hat) || !a4(delta_v))))
    return SAGE_ERR_MISALIGNED;
  if ((s = check_device()) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = static_cast<size_t>(B) * H_kv * sage::stat_chunks(N) * d;
  void* scratch = nullptr;
  cudaError_t e = cudaMallocAsync(&scratch, n * 12, st);
  if (e != cudaSuccess) {
    sage::set_error_detail("cudaMallocAsync(scratch)", e);
    return from_cuda(e);
  }
  long long* ksum = static_cast<long long*>(scratch);
  uint32_t* vmax = reinterpret_cast<uint32_t*>(ksum + n);
  e = run_prepass(q, k, v, B, H, H_kv, N, d, sm_scale, v_r, q_hat, k_hat, v_hat, delta_q, delta_k,
                  mean_k, delta_v, ksum, vmax, st);
  cudaError_t ef = cudaFreeAsync(scratch, st);
  return from_cuda(e != cudaSuccess ? e : ef);
}

sage_status_t sage_smooth_quant_qkv_rope(const void* q, const void* k, const void* v,
                                         const float* cos_t, const float* sin_t, int B, int H,
                                         int H_kv, int N, int d, float sm_scale, float v_r,
                                         int8_t* q_hat, int8_t* k_hat, uint8_t* v_hat,
                                         float* delta_q, float* delta_k, float* mean_k,
                                         float* delta_v, void* stream) {
  sage_status_t s = check_sizes(B, H, H_kv, N, d);
  if (s != SAGE_OK) return s;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  const bool hv = v != nullptr;
  if (hv && (!(v_r > 0.f) || !(v_r <= 448.f))) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return SAGE_OK;
  if (!q || !k || !cos_t || !sin_t || !q_hat || !k_hat || !delta_q || !delta_k || !mean_k)
    return SAGE_ERR_INVALID_ARG;
  if (hv != (v_hat != nullptr) || hv != (delta_v != nullptr)) return SAGE_ERR_INVALID_ARG;
  if (!a16(q) || !a16(k) || !a16(cos_t) || !a16(sin_t) || !a16(q_hat) || !a16(k_hat) ||
      !a4(delta_q) || !a4(delta_k) || !a4(mean_k) || (hv && (!a16(v) || !a16(v_hat) || !a4(delta_v))))
    return SAGE_ERR_MISALIGNED;
  if ((s = check_device()) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = static_cast<size_t>(B) * H_kv * sage::stat_chunks(N) * d;
  void* scratch = nullptr;
  cudaError_t e = cudaMallocAsync(&scratch, n * 12, st);
  if (e != cudaSuccess) {
    sage::set_error_detail("cudaMallocAsync(scratch)", e);
    return from_cuda(e);
  }
  long long* ksum = static_cast<long long*>(scratch);
  uint32_t* vmax = reinterpret_cast<uint32_t*>(ksum + n);
  e = run_prepass(q, k, v, B, H, H_kv, N, d, sm_scale, v_r, q_hat, k_hat, v_hat, delta_q, delta_k,
                  mean_k, delta_v, ksum, vmax, st, cos_t, sin_t);
  cudaError_t ef = cudaFreeAsync(scratch, st);
  return from_cuda(e != cudaSuccess ? e : ef);
}

sage_status_t sage_attn_fwd_quantized(const int8_t* q_hat, const int8_t* k_hat,
                                      const float* delta_q, const float* delta_k,
                                      const void* v_or_vhat, const float* delta_v, void* o, int B,
                                      int H, int H_kv, int N, int d, int causal, int variant,
                                      void* stream) {
  sage_status_t s = check_sizes(B, H, H_kv, N, d);
  if (s != SAGE_OK) return s;
  if (variant != SAGE_VARIANT_B && variant != SAGE_VARIANT_8P8 && variant != SAGE_VARIANT_8P8_R56)
    return SAGE_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return SAGE_OK;
  if (!q_hat || !k_hat || !delta_q || !delta_k || !v_or_vhat || !o) return SAGE_ERR_INVALID_ARG;
  if (variant != SAGE_VARIANT_B && !delta_v) return SAGE_ERR_INVALID_ARG;
  if (!a16(q_hat) || !a16(k_hat) || !a16(v_or_vhat) || !a16(o) || !a4(delta_q) || !a4(delta_k) ||
      (delta_v && !a4(delta_v)))
    return SAGE_ERR_MISALIGNED;
  if ((s = check_device()) != SAGE_OK) return s;
  sage::AttnArgs aa;
  aa.q_hat = q_hat;
  aa.k_hat = k_hat;
  aa.delta_q = delta_q;
  aa.delta_k = delta_k;
  aa.v = v_or_vhat;
  aa.delta_v = delta_v;
  aa.o = o;
  aa.B = B;
  aa.H = H;
  aa.H_kv = H_kv;
  aa.N = N;
  aa.d = d;
  aa.causal = causal;
  aa.variant = variant == SAGE_VARIANT_B ? 0 : 1;
  aa.p_r = variant == SAGE_VARIANT_8P8_R56 ? 56.f : 448.f;
  aa.timeout_ns = g_timeout_ns.load();
  return from_cuda(sage::launch_attention(aa, static_cast<cudaStream_t>(stream)));
}

size_t sage_attn_workspace_bytes(int B, int H, int H_kv, int N, int d, int variant) {
  if (check_sizes(B, H, H_kv, N, d) != SAGE_OK || B == 0 || N == 0) return 0;
  return ws_layout(B, H, H_kv, N, d, variant).total;
}

sage_status_t sage_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, int B, int H,
                               int H_kv, int N, int d, int causal, float sm_scale, int variant,
                               void* workspace, size_t ws_bytes, void* stream) {
  sage_status_t s = check_fwd_args(q, k, v, o, B, H, H_kv, N, d, causal, sm_scale, variant);
  if (s != SAGE_OK || B == 0 || N == 0) return s;
  if ((s = check_device()) != SAGE_OK) return s;
  const WsLayout L = ws_layout(B, H, H_kv, N, d, variant);
  if (workspace == nullptr || ws_bytes < L.total) return SAGE_ERR_NO_MEMORY;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SAGE_ERR_MISALIGNED;
  return run_forward(q, k, v, o, B, H, H_kv, N, d, causal, sm_scale, variant,
                     static_cast<uint8_t*>(workspace), L, static_cast<cudaStream_t>(stream));
}

sage_status_t sage_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H,
                            int H_kv, int N, int d, int causal, float sm_scale, int variant,
                            void* stream) {
  sage_status_t s = check_fwd_args(q, k, v, o, B, H, H_kv, N, d, causal, sm_scale, variant);
  if (s != SAGE_OK || B == 0 || N == 0) return s;
  if ((s = check_device()) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(B, H, H_kv, N, d, variant);
  void* ws = nullptr;
  cudaError_t e = cudaMallocAsync(&ws, L.total, st);
  if (e != cudaSuccess) {
    sage::set_error_detail("cudaMallocAsync(workspace)", e);
    return from_cuda(e);
  }
  s = run_forward(q, k, v, o, B, H, H_kv, N, d, causal, sm_scale, variant,
                  static_cast<uint8_t*>(ws), L, st);
  cudaError_t ef = cudaFreeAsync(ws, st);
  if (s != SAGE_OK) return s;
  return from_cuda(ef);
}

namespace {

// Side streams and events of sage_attn_fwd_host, created once per device
// and reused by the call that holds the device's lock; a concurrent call on
// the same device makes its own and destroys them afterwards.
constexpr int kHostChunks = 8;
struct HostPipe {
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev[2 * kHostChunks + 2] = {};
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu[kMaxDevices];

cudaError_t pipe_create(HostPipe* P) {
  cudaError_t e = cudaStreamCreateWithFlags(&P->s_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&P->s_out, cudaStreamNonBlocking);
  for (int i = 0; e == cudaSuccess && i < 2 * kHostChunks + 2; ++i)
    e = cudaEventCreateWithFlags(&P->ev[i], cudaEventDisableTiming);
  return e;
}

void pipe_destroy(HostPipe* P) {
  for (int i = 0; i < 2 * kHostChunks + 2; ++i)
    if (P->ev[i]) cudaEventDestroy(P->ev[i]);
  if (P->s_in) cudaStreamDestroy(P->s_in);
  if (P->s_out) cudaStreamDestroy(P->s_out);
  *P = HostPipe();
}

}  // namespace

sage_status_t sage_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                                 void* o_host, int B, int H, int H_kv, int N, int d, int causal,
                                 float sm_scale, int variant, void* stream) {
  sage_status_t s = check_sizes(B, H, H_kv, N, d);
  if (s != SAGE_OK) return s;
  if (variant != SAGE_VARIANT_B && variant != SAGE_VARIANT_8P8 && variant != SAGE_VARIANT_8P8_R56)
    return SAGE_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || N == 0) return SAGE_OK;
  if (!q_host || !k_host || !v_host || !o_host) return SAGE_ERR_INVALID_ARG;
  if ((s = check_device()) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // The problem splits into independent units, one per (batch, kv head) with
  // its group of query heads; consecutive units are contiguous in every
  // tensor.  Chunks of units are pipelined: copies in on one stream, the
  // pass on `stream`, copies out on a third, so the transfers of one chunk
  // overlap the kernels of another.
  constexpr int kMaxChunks = kHostChunks;
  const int units = B * H_kv, r = H / H_kv;
  const int nchunk = units < kMaxChunks ? units : kMaxChunks;
  const int per = (units + nchunk - 1) / nchunk;
  const size_t qu = static_cast<size_t>(r) * N * d * 2;  // bytes of one unit of q (and o)
  const size_t ku = static_cast<size_t>(N) * d * 2;      // bytes of one unit of k (and v)
  const size_t qb = qu * units, kb = ku * units;
  const WsLayout L = ws_layout(1, per * r, per, N, d, variant);
  const size_t off_k = align256(qb), off_v = off_k + align256(kb), off_o = off_v + align256(kb);
  const size_t off_ws = off_o + align256(qb);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);  // in [0, kMaxDevices): check_device passed
  if (e != cudaSuccess) return from_cuda(e);
  std::unique_lock<std::mutex> lock(g_pipe_mu[dev], std::try_to_lock);
  HostPipe own;
  HostPipe* P = lock.owns_lock() ? &g_pipe[dev] : &own;
  if (P->s_in == nullptr) {
    e = pipe_create(P);
    if (e != cudaSuccess) {
      pipe_destroy(P);
      sage::set_error_detail("sage_attn_fwd_host streams", e);
      return from_cuda(e);
    }
  }
  cudaStream_t s_in = P->s_in, s_out = P->s_out;
  cudaEvent_t* ev = P->ev;
  cudaEvent_t* ev_in = ev;               // [nchunk] inputs of chunk c on the device
  cudaEvent_t* ev_done = ev + nchunk;    // [nchunk] output of chunk c computed
  cudaEvent_t ev_alloc = ev[2 * nchunk], ev_out = ev[2 * nchunk + 1];

  void* buf = nullptr;
  bool allocated = false;
  if (e == cudaSuccess) e = cudaMallocAsync(&buf, off_ws + L.total, st);
  if (e == cudaSuccess) {
    allocated = true;
    e = cudaEventRecord(ev_alloc, st);
  }
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev_alloc, 0);
  uint8_t* base = static_cast<uint8_t*>(buf);
  const uint8_t* hq = static_cast<const uint8_t*>(q_host);
  const uint8_t* hk = static_cast<const uint8_t*>(k_host);
  const uint8_t* hv = static_cast<const uint8_t*>(v_host);
  uint8_t* ho = static_cast<uint8_t*>(o_host);
  for (int c = 0; e == cudaSuccess && c < nchunk; ++c) {
    const int u0 = c * per, n = (units - u0 < per ? units - u0 : per);
    if (n <= 0) break;
    e = cudaMemcpyAsync(base + u0 * qu, hq + u0 * qu, n * qu, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + off_k + u0 * ku, hk + u0 * ku, n * ku, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + off_v + u0 * ku, hv + u0 * ku, n * ku, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in[c], s_in);
  }
  for (int c = 0; e == cudaSuccess && s == SAGE_OK && c < nchunk; ++c) {
    const int u0 = c * per, n = (units - u0 < per ? units - u0 : per);
    if (n <= 0) break;
    e = cudaStreamWaitEvent(st, ev_in[c], 0);
    if (e != cudaSuccess) break;
    s = run_forward(base + u0 * qu, base + off_k + u0 * ku, base + off_v + u0 * ku,
                    base + off_o + u0 * qu, 1, n * r, n, N, d, causal, sm_scale, variant,
                    base + off_ws, ws_layout(1, n * r, n, N, d, variant), st);
    if (s == SAGE_OK) e = cudaEventRecord(ev_done[c], st);
    if (e == cudaSuccess && s == SAGE_OK) e = cudaStreamWaitEvent(s_out, ev_done[c], 0);
    if (e == cudaSuccess && s == SAGE_OK)
      e = cudaMemcpyAsync(ho + u0 * qu, base + off_o + u0 * qu, n * qu, cudaMemcpyDeviceToHost, s_out);
  }
  // everything on the side streams ends before the buffer is freed on `stream`
  cudaError_t ec = cudaSuccess;
  if (s_in) ec = cudaStreamSynchronize(s_in);
  if (s_out && ec == cudaSuccess) ec = cudaEventRecord(ev_out, s_out);
  if (s_out && ec == cudaSuccess) ec = cudaStreamWaitEvent(st, ev_out, 0);
  cudaError_t ef = allocated ? cudaFreeAsync(buf, st) : cudaSuccess;
  cudaError_t es = cudaStreamSynchronize(st);
  if (s_out) cudaStreamSynchronize(s_out);
  if (P == &own) pipe_destroy(&own);
  if (s != SAGE_OK) return s;
  if (e != cudaSuccess) {
    sage::set_error_detail("sage_attn_fwd_host pipeline", e);
    return from_cuda(e);
  }
  if (ec != cudaSuccess) return from_cuda(ec);
  if (ef != cudaSuccess) return from_cuda(ef);
  return from_cuda(es);
}

// ------------------------------------------------ packed variable-length batches
namespace {

sage_status_t check_varlen(const int32_t* cu, int B, int max_seqlen, int T, int H, int H_kv, int d) {
  sage_status_t s = check_sizes(B, H, H_kv, max_seqlen, d);
  if (s != SAGE_OK) return s;
  if (T < 0) return SAGE_ERR_INVALID_ARG;
  if (T > (1 << 30)) return SAGE_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
  if (B > 0 && T > 0 && max_seqlen > 0 && cu == nullptr) return SAGE_ERR_INVALID_ARG;
  if (cu != nullptr && !a4(cu)) return SAGE_ERR_MISALIGNED;
  return SAGE_OK;
}

sage::SeqLayout packed(const int32_t* cu, int max_seqlen, int T) {
  sage::SeqLayout L;
  L.cu = cu;
  L.T = T;
  L.max_len = max_seqlen;
  return L;
}

}  // namespace

sage_status_t sage_smooth_quant_qkv_varlen(const void* q, const void* k, const void* v,
                                           const int32_t* cu_seqlens, int B, int max_seqlen, int T,
                                           int H, int H_kv, int d, float sm_scale, float v_r,
                                           int8_t* q_hat, int8_t* k_hat, uint8_t* v_hat,
                                           float* delta_q, float* delta_k, float* mean_k,
                                           float* delta_v, void* stream) {
  sage_status_t s = check_varlen(cu_seqlens, B, max_seqlen, T, H, H_kv, d);
  if (s != SAGE_OK) return s;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  const bool hv = v != nullptr;
  if (hv && (!(v_r > 0.f) || !(v_r <= 448.f))) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || T == 0 || max_seqlen == 0) return SAGE_OK;
  if (!q || !k || !q_hat || !k_hat || !delta_q || !delta_k || !mean_k) return SAGE_ERR_INVALID_ARG;
  if (hv != (v_hat != nullptr) || hv != (delta_v != nullptr)) return SAGE_ERR_INVALID_ARG;
  if (!a16(q) || !a16(k) || !a16(q_hat) || !a16(k_hat) || !a4(delta_q) || !a4(delta_k) ||
      !a4(mean_k) || (hv && (!a16(v) || !a16(v_hat) || !a4(delta_v))))
    return SAGE_ERR_MISALIGNED;
  if ((s = check_device()) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = static_cast<size_t>(B) * H_kv * sage::stat_chunks(max_seqlen) * d;
  void* scratch = nullptr;
  cudaError_t e = cudaMallocAsync(&scratch, n * 12, st);
  if (e != cudaSuccess) {
    sage::set_error_detail("cudaMallocAsync(scratch)", e);
    return from_cuda(e);
  }
  long long* ksum = static_cast<long long*>(scratch);
  uint32_t* vmax = reinterpret_cast<uint32_t*>(ksum + n);
  e = run_prepass(q, k, v, B, H, H_kv, max_seqlen, d, sm_scale, v_r, q_hat, k_hat, v_hat, delta_q,
                  delta_k, mean_k, delta_v, ksum, vmax, st, nullptr, nullptr,
                  packed(cu_seqlens, max_seqlen, T));
  cudaError_t ef = cudaFreeAsync(scratch, st);
  return from_cuda(e != cudaSuccess ? e : ef);
}

sage_status_t sage_attn_fwd_varlen_quantized(const int8_t* q_hat, const int8_t* k_hat,
                                             const float* delta_q, const float* delta_k,
                                             const void* v_or_vhat, const float* delta_v, void* o,
                                             const int32_t* cu_seqlens, int B, int max_seqlen, int T,
                                             int H, int H_kv, int d, int causal, int variant,
                                             void* stream) {
  sage_status_t s = check_varlen(cu_seqlens, B, max_seqlen, T, H, H_kv, d);
  if (s != SAGE_OK) return s;
  if (variant != SAGE_VARIANT_B && variant != SAGE_VARIANT_8P8 && variant != SAGE_VARIANT_8P8_R56)
    return SAGE_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || T == 0 || max_seqlen == 0) return SAGE_OK;
  if (!q_hat || !k_hat || !delta_q || !delta_k || !v_or_vhat || !o) return SAGE_ERR_INVALID_ARG;
  if (variant != SAGE_VARIANT_B && !delta_v) return SAGE_ERR_INVALID_ARG;
  if (!a16(q_hat) || !a16(k_hat) || !a16(v_or_vhat) || !a16(o) || !a4(delta_q) || !a4(delta_k) ||
      (delta_v && !a4(delta_v)))
    return SAGE_ERR_MISALIGNED;
  if ((s = check_device()) != SAGE_OK) return s;
  sage::AttnArgs aa;
  aa.q_hat = q_hat;
  aa.k_hat = k_hat;
  aa.delta_q = delta_q;
  aa.delta_k = delta_k;
  aa.v = v_or_vhat;
  aa.delta_v = delta_v;
  aa.o = o;
  aa.B = B;
  aa.H = H;
  aa.H_kv = H_kv;
  aa.N = max_seqlen;
  aa.d = d;
  aa.causal = causal;
  aa.variant = variant == SAGE_VARIANT_B ? 0 : 1;
  aa.p_r = variant == SAGE_VARIANT_8P8_R56 ? 56.f : 448.f;
  aa.timeout_ns = g_timeout_ns.load();
  aa.cu = cu_seqlens;
  aa.T = T;
  return from_cuda(sage::launch_attention(aa, static_cast<cudaStream_t>(stream)));
}

sage_status_t sage_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                                   const int32_t* cu_seqlens, int B, int max_seqlen, int T, int H,
                                   int H_kv, int d, int causal, float sm_scale, int variant,
                                   void* stream) {
  sage_status_t s = check_varlen(cu_seqlens, B, max_seqlen, T, H, H_kv, d);
  if (s != SAGE_OK) return s;
  if (variant != SAGE_VARIANT_B && variant != SAGE_VARIANT_8P8 && variant != SAGE_VARIANT_8P8_R56)
    return SAGE_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return SAGE_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if (B == 0 || T == 0 || max_seqlen == 0) return SAGE_OK;
  if (!q || !k || !v || !o) return SAGE_ERR_INVALID_ARG;
  if (!a16(q) || !a16(k) || !a16(v) || !a16(o)) return SAGE_ERR_MISALIGNED;
  if ((s = check_device()) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(B, H, H_kv, max_seqlen, d, variant, T);
  void* ws = nullptr;
  cudaError_t e = cudaMallocAsync(&ws, L.total, st);
  if (e != cudaSuccess) {
    sage::set_error_detail("cudaMallocAsync(workspace)", e);
    return from_cuda(e);
  }
  s = run_forward(q, k, v, o, B, H, H_kv, max_seqlen, d, causal, sm_scale, variant,
                  static_cast<uint8_t*>(ws), L, st, packed(cu_seqlens, max_seqlen, T));
  cudaError_t ef = cudaFreeAsync(ws, st);
  if (s != SAGE_OK) return s;
  return from_cuda(ef);
}

int sage_v_hat_layout(void) { return 0; }

sage_status_t sage_get_device_error(void* stream, uint32_t* detail) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SAGE_ERR_CUDA;
  uint32_t w = 0;
  if (sage::read_and_clear_error(&w) != cudaSuccess) return SAGE_ERR_CUDA;
  if (detail) *detail = w;
  return (w & sage::ERR_TIMEOUT) ? SAGE_ERR_DEVICE_TIMEOUT : SAGE_OK;
}

void sage_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns == 0 ? 1 : ns); }

sage_status_t sage_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  sage_status_t s = check_device();
  if (s != SAGE_OK) return s;
  return from_cuda(sage::launch_selftest_wait(timeout_ns, static_cast<cudaStream_t>(stream)));
}

const char* sage_status_string(sage_status_t status) {
  switch (status) {
    case SAGE_OK: return "ok";
    case SAGE_ERR_INVALID_ARG: return "invalid argument";
    case SAGE_ERR_UNSUPPORTED: return "unsupported shape or variant";
    case SAGE_ERR_MISALIGNED: return "pointer not aligned";
    case SAGE_ERR_DEVICE: return "current device is not a B200 (compute capability 10.0)";
    case SAGE_ERR_CUDA: return "CUDA call failed";
    case SAGE_ERR_DEVICE_TIMEOUT: return "a kernel abandoned a bounded wait";
    case SAGE_ERR_NO_MEMORY: return "out of device memory or workspace too small";
  }
  return "unknown status";
}

const char* sage_version(void) { return "0.1.0"; }

const char* sage_last_error_detail(void) { return sage::error_detail(); }

}  // extern "C"
