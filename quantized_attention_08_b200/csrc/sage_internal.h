// sage_internal.h -- declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sage_ptx.cuh"

namespace sage {

// Where the token rows of a slab live.  A slab is one head of one sequence,
// numbered z = b * Hs + h (Hs = heads of that tensor: H for Q and O, H_kv for
// K and V).  Fixed layout ([B, Hs, N, d]): slab z holds rows z*N .. z*N + N-1.
// Packed variable-length layout ([Hs, T, d]; sequence b holds tokens
// cu[b] .. cu[b+1]-1 of every head): slab z holds rows h*T + cu[b] onward,
// len_b = cu[b+1] - cu[b] of them.  Offsets are clamped to [0, T] and
// lengths to max_len, so malformed offsets cannot reach outside the tensor.
struct SeqLayout {
  const int* cu = nullptr;  // device [B+1] token offsets, or nullptr (fixed layout)
  int T = 0;                // fixed: N; packed: total tokens
  int max_len = 0;          // fixed: N; packed: bound on every len_b
};

#if defined(__CUDACC__)
__device__ __forceinline__ void slab_rows(const SeqLayout& L, int z, int Hs, size_t* row0, int* len) {
  if (L.cu == nullptr) {
    *row0 = static_cast<size_t>(z) * L.T;
    *len = L.T;
    return;
  }
  const int b = z / Hs, h = z % Hs;
  int a = L.cu[b], e = L.cu[b + 1];
  a = a < 0 ? 0 : (a > L.T ? L.T : a);
  e = e < a ? a : (e > L.T ? L.T : e);
  *row0 = static_cast<size_t>(h) * L.T + a;
  *len = (e - a) < L.max_len ? (e - a) : L.max_len;
}
#endif

struct QuantArgs {
  const void* q;        // fp16 [B,H,N,d] or nullptr
  const void* k;        // fp16 [B,Hkv,N,d] or nullptr
  const void* v;        // fp16 [B,Hkv,N,d] or nullptr (8+8 only)
  int8_t* q_hat;
  int8_t* k_hat;
  uint8_t* v_hat;
  float* delta_q;
  float* delta_k;
  const float* mean_k;
  const float* delta_v;
  float sm_scale;
  int B, H, H_kv, N, d;
  const float* cos_t = nullptr;  // rotary tables [N, d/2] fp32, or nullptr
  const float* sin_t = nullptr;
  SeqLayout seq;                 // seq.cu == nullptr: fixed layout with N rows per slab
};

size_t stat_chunks(int N);
// slabs = B * H_kv; N rows per slab (fixed layout) or at most seq.max_len
// (packed layout, seq.cu != nullptr; N is then seq.max_len)
cudaError_t launch_colstats(const void* k, const void* v, int slabs, int N, int D, long long* ksum,
                            uint32_t* vmax, cudaStream_t st, const float* cos_t = nullptr,
                            const float* sin_t = nullptr, SeqLayout seq = SeqLayout(), int Hkv = 1);
cudaError_t launch_finalize(const long long* ksum, const uint32_t* vmax, int slabs, int N, int D,
                            float v_r, float* mean_k, float* delta_v, cudaStream_t st,
                            SeqLayout seq = SeqLayout(), int Hkv = 1);
cudaError_t launch_quant(const QuantArgs& a, cudaStream_t st);

struct AttnArgs {
  const int8_t* q_hat;
  const int8_t* k_hat;
  const float* delta_q;
  const float* delta_k;
  const void* v;         // fp16 V (variant B) or e4m3 codes (8+8)
  const float* delta_v;  // 8+8 only
  void* o;               // fp16 [B,H,N,d]
  int B, H, H_kv, N, d, causal, variant;  // variant: 0 = fp16 P~V, 1 = e4m3 P~V
  uint64_t timeout_ns;
  float p_r = 448.f;  // e4m3 P operand = p_r * P~ (variant 1)
  // packed sequences (cu != nullptr): q, o are [H, T, d], k, v [H_kv, T, d],
  // sequence b at tokens cu[b] .. cu[b+1]-1; N is the longest allowed length
  // and B the number of sequences
  const int* cu = nullptr;
  int T = 0;
};

// Returns a cudaError_t; CUDA_ERROR codes of tensor-map encoding are mapped
// to cudaErrorInvalidValue.
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st);

cudaError_t launch_selftest_wait(uint64_t timeout_ns, cudaStream_t st);
cudaError_t read_and_clear_error(uint32_t* word);

// Records a human-readable description of the last failing step of this
// thread's most recent call (see sage_last_error_detail()).
void set_error_detail(const char* step, cudaError_t e, int extra = 0);
const char* error_detail();

}  // namespace sage
