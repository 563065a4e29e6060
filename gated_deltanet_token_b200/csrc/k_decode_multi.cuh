// k_decode_multi.cuh -- K decode tokens per sequence in one pass over the state (K <= 8).
//
// Same per-token rule as k_decode (field guide §02, steps 1-6, then the gated RMSNorm), applied
// to K consecutive tokens of each sequence.  The state rows stay in registers across the K
// tokens, so each 512-byte row is read once and written once per call instead of once per
// token.  Conv: the K new raw rows follow the three history rows; the history keeps the last
// three raw rows.  One CTA per (sequence n, QK head j) as in k_decode.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int DECM_KMAX = 8;
constexpr int DECM_ROWS = 4;  // state rows in flight per warp (x K tokens of dot products)

// smem: q, k [KMAX][D]; v, y [KMAX][GMAX=8][D]; gates [KMAX][8] x 2; kq [KMAX]
template <bool BF16, bool OUT_BF16>
__global__ void __launch_bounds__(256) k_decode_multi(Dims d, int K, const void* __restrict__ q,
                                                      const void* __restrict__ k, const void* __restrict__ v,
                                                      const void* __restrict__ z, const float* __restrict__ a,
                                                      const float* __restrict__ b, const float* __restrict__ A_log,
                                                      const float* __restrict__ dt_bias,
                                                      const float* __restrict__ conv_w,
                                                      const float* __restrict__ norm_w, void* conv_state,
                                                      float* state, void* __restrict__ y) {
  using E = typename std::conditional<BF16, uint16_t, float>::type;
  const int n = blockIdx.x, j = blockIdx.y;
  const int hq = d.h_qk, hv = d.h_v, G = hv / hq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t cconv = (size_t)(2 * hq + hv) * D;
  extern __shared__ __align__(16) float dm[];
  float* qs = dm;                                 // [KMAX][D]
  float* ks = qs + DECM_KMAX * D;                 // [KMAX][D]
  float* vs = ks + DECM_KMAX * D;                 // [KMAX][8][D]
  float* ys = vs + DECM_KMAX * 8 * D;             // [KMAX][8][D]
  float* al = ys + DECM_KMAX * 8 * D;             // [KMAX][8]
  float* be = al + DECM_KMAX * 8;                 // [KMAX][8]
  float* kqv = be + DECM_KMAX * 8;                // [KMAX]
  if (K < 1 || K > DECM_KMAX || G > 8) {
    if (tid == 0) atomicExch(&g_gdn_status, -6);
    return;
  }

  // conv + SiLU for the K tokens over this CTA's channels; the history becomes the last
  // three raw rows of (history, new rows), copied exactly
  E* cs = static_cast<E*>(conv_state) + (size_t)n * 3 * cconv;
  const int nch = 2 * D + G * D;
  for (int c = tid; c < nch; c += blockDim.x) {
    size_t ch;
    const E* src;  // token t's raw value at src[t * stride]
    size_t stride;
    float* dst;    // token t's output at dst[t * dstride]
    int dstride;
    if (c < D) {
      ch = (size_t)j * D + c;
      src = static_cast<const E*>(q) + ((size_t)n * K * hq + j) * D + c;
      stride = (size_t)hq * D;
      dst = qs + c;
      dstride = D;
    } else if (c < 2 * D) {
      ch = (size_t)(hq + j) * D + (c - D);
      src = static_cast<const E*>(k) + ((size_t)n * K * hq + j) * D + (c - D);
      stride = (size_t)hq * D;
      dst = ks + (c - D);
      dstride = D;
    } else {
      const int g = (c - 2 * D) / D, cc = (c - 2 * D) % D, hh = j * G + g;
      ch = (size_t)2 * hq * D + (size_t)hh * D + cc;
      src = static_cast<const E*>(v) + ((size_t)n * K * hv + hh) * D + cc;
      stride = (size_t)hv * D;
      dst = vs + g * D + cc;
      dstride = 8 * D;
    }
    const float4 w = *reinterpret_cast<const float4*>(conv_w + ch * 4);
    E win[3] = {cs[ch], cs[cconv + ch], cs[2 * cconv + ch]};  // x_{-3}, x_{-2}, x_{-1}
    for (int t = 0; t < K; ++t) {
      const E xin = src[(size_t)t * stride];
      float f0, f1, f2, f3;
      if constexpr (BF16) {
        f0 = bf2f(win[0]); f1 = bf2f(win[1]); f2 = bf2f(win[2]); f3 = bf2f(xin);
      } else {
        f0 = win[0]; f1 = win[1]; f2 = win[2]; f3 = xin;
      }
      dst[t * dstride] = silu_f(fmaf(w.w, f3, fmaf(w.z, f2, fmaf(w.y, f1, w.x * f0))));
      win[0] = win[1]; win[1] = win[2]; win[2] = xin;
    }
    cs[ch] = win[0];
    cs[cconv + ch] = win[1];
    cs[2 * cconv + ch] = win[2];
  }
  for (int i = tid; i < K * G; i += blockDim.x) {
    const int t = i / G, g = i % G, hh = j * G + g;
    const size_t o = ((size_t)n * K + t) * hv + hh;
    al[t * 8 + g] = expf(decay_gate_f(a[o], A_log[hh], dt_bias[hh]));
    be[t * 8 + g] = sigmoid_f(b[o]);
  }
  __syncthreads();
  for (int i = warp; i < 2 * K; i += 8) {  // L2 norms: q_t (times q_scale) and k_t
    const int t = i >> 1, isk = i & 1;
    float* p = (isk ? ks : qs) + t * D;
    float4 x = *reinterpret_cast<float4*>(p + lane * 4);
    const float ss = warp_sum(x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w);
    const float inv = (isk ? 1.0f : d.q_scale) / sqrtf(ss + d.l2_eps);
    x.x *= inv; x.y *= inv; x.z *= inv; x.w *= inv;
    *reinterpret_cast<float4*>(p + lane * 4) = x;
  }
  __syncthreads();
  for (int t = warp; t < K; t += 8) {
    const float4 kr = *reinterpret_cast<const float4*>(ks + t * D + lane * 4);
    const float4 qr = *reinterpret_cast<const float4*>(qs + t * D + lane * 4);
    const float s = warp_sum(dot4(kr, qr));
    if (lane == 0) kqv[t] = s;
  }
  __syncthreads();

  // state rows: an equal contiguous share per warp, DECM_ROWS in flight, K tokens each
  const int rows_per_warp = G * D / 8;
  const size_t state0 = ((size_t)n * hv + (size_t)j * G) * D * D;
  for (int r0 = warp * rows_per_warp; r0 < (warp + 1) * rows_per_warp; r0 += DECM_ROWS) {
    float4 s[DECM_ROWS];
#pragma unroll
    for (int u = 0; u < DECM_ROWS; ++u)
      s[u] = __ldcs(reinterpret_cast<const float4*>(state + state0 + (size_t)(r0 + u) * D + lane * 4));
    for (int t = 0; t < K; ++t) {
      const float4 kr = *reinterpret_cast<const float4*>(ks + t * D + lane * 4);
      const float4 qr = *reinterpret_cast<const float4*>(qs + t * D + lane * 4);
      const float kq = kqv[t];
#pragma unroll
      for (int u = 0; u < DECM_ROWS; ++u) {
        const int row = r0 + u, g = row / D, i = row % D;
        const float rk = warp_sum(dot4(s[u], kr));
        const float rq = warp_sum(dot4(s[u], qr));
        const float a_ = al[t * 8 + g];
        const float e = be[t * 8 + g] * (vs[(t * 8 + g) * D + i] - a_ * rk);
        s[u].x = fmaf(a_, s[u].x, e * kr.x);
        s[u].y = fmaf(a_, s[u].y, e * kr.y);
        s[u].z = fmaf(a_, s[u].z, e * kr.z);
        s[u].w = fmaf(a_, s[u].w, e * kr.w);
        if (lane == 0) ys[(t * 8 + g) * D + i] = fmaf(a_, rq, e * kq);
      }
    }
#pragma unroll
    for (int u = 0; u < DECM_ROWS; ++u)
      __stcs(reinterpret_cast<float4*>(state + state0 + (size_t)(r0 + u) * D + lane * 4), s[u]);
  }
  __syncthreads();
  for (int i = warp; i < K * G; i += 8) {  // gated RMSNorm of each (token, value head)
    const int t = i / G, g = i % G;
    const float4 yv = *reinterpret_cast<const float4*>(ys + (t * 8 + g) * D + lane * 4);
    const float ss = warp_sum(yv.x * yv.x + yv.y * yv.y + yv.z * yv.z + yv.w * yv.w);
    const float inv = 1.0f / sqrtf(ss * (1.0f / D) + d.rms_eps);
    const size_t off = (((size_t)n * K + t) * hv + (size_t)j * G + g) * D + lane * 4;
    const float4 zz = load4<BF16>(z, off);
    const float4 nw = *reinterpret_cast<const float4*>(norm_w + lane * 4);
    float4 o;
    o.x = yv.x * inv * nw.x * silu_f(zz.x);
    o.y = yv.y * inv * nw.y * silu_f(zz.y);
    o.z = yv.z * inv * nw.z * silu_f(zz.z);
    o.w = yv.w * inv * nw.w * silu_f(zz.w);
    store4<OUT_BF16>(y, off, o);
  }
}

constexpr size_t DECM_SMEM = (size_t)(2 * DECM_KMAX * D + 2 * DECM_KMAX * 8 * D + 2 * DECM_KMAX * 8 + DECM_KMAX) * 4;

}  // namespace gdn
