// gdn_common.cuh -- shared device helpers of the sm_100a GDN kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

constexpr int D = 128;  // head width: d_k = d_v = 128 (the pages' model; the only width supported)
constexpr int CH = 64;  // chunk length of the chunked prefill

// Kernel-side view of the public gdn_dims_t.
struct Dims {
  int n_seqs, total_tokens, h_qk, h_v;
  int in_bf16, out_bf16;
  float q_scale, l2_eps, rms_eps;
};

// One chunk of the varlen tile map: chunks start at each sequence's first token and the
// last chunk of a sequence is partial.  len == 0 marks an unused slot.
struct __align__(16) ChunkEntry {
  int seq;        // sequence index
  int t0;         // first packed token of the chunk
  int len;        // tokens in the chunk, 0..64
  int seq_start;  // first packed token of the sequence (conv history stops there)
};

// Entry c of the tile map.  With no table (tab == nullptr: one sequence of `total` tokens)
// the entry is computed: chunk c covers tokens 64 c .. 64 c + 63 of sequence 0.
__device__ __forceinline__ ChunkEntry chunk_entry(const ChunkEntry* tab, int total, int c) {
  if (tab) return tab[c];
  ChunkEntry e;
  e.seq = 0;
  e.t0 = c * 64;
  e.len = min(64, max(0, total - c * 64));
  e.seq_start = 0;
  return e;
}

__device__ __forceinline__ float bf2f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

__device__ __forceinline__ uint16_t f2bf(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Four consecutive elements starting at element index i (i % 4 == 0) as fp32.
template <bool BF16>
__device__ __forceinline__ float4 load4(const void* p, size_t i) {
  if constexpr (BF16) {
    const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p) + i);
    return make_float4(bf2f(u.x & 0xffffu), bf2f(u.x >> 16), bf2f(u.y & 0xffffu), bf2f(u.y >> 16));
  } else {
    return *reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
  }
}

template <bool BF16>
__device__ __forceinline__ void store4(void* p, size_t i, float4 v) {
  if constexpr (BF16) {
    uint2 u;
    u.x = uint32_t(f2bf(v.x)) | (uint32_t(f2bf(v.y)) << 16);
    u.y = uint32_t(f2bf(v.z)) | (uint32_t(f2bf(v.w)) << 16);
    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p) + i) = u;
  } else {
    *reinterpret_cast<float4*>(static_cast<float*>(p) + i) = v;
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }
// Hardware-approximate forms (ex2.approx, rcp.approx: a few ulp per factor) for the
// streaming kernels of the bf16 path and the output gate, where operand rounding (bf16 hi/lo
// products, ~2^-17) or the output tolerance dominates by orders of magnitude.  For x far
// below zero e^-x overflows and the quotient goes to 0, the limit of silu and sigmoid.
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
__device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float softplus_f(float x) {
  return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}
// Decay gate ("Qwen3.8-Flash-Next" model notes, decay-gate note):
// g = -exp(A_log) * softplus(a + dt_bias).
__device__ __forceinline__ float decay_gate_f(float a, float A_log, float dt_bias) {
  return -expf(A_log) * softplus_f(a + dt_bias);
}

// Component c (compile-time after unrolling) of a float4.
__device__ __forceinline__ float comp(const float4& v, int c) {
  return c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

// Library-wide device status word: a bounded device-side wait that gives up records its
// error code here (read and cleared by gdn_read_device_status).
__device__ int g_gdn_status = 0;

}  // namespace gdn
