// k_decode.cuh -- one decode step on resident states (K4).
//
// For each (sequence n, QK head j) one CTA handles the G = h_v / h_qk value heads that
// share QK head j, so the q/k conv history of that head is read and shifted by exactly
// one CTA.  Per token: width-4 causal conv on the raw history (conv_state) plus the new
// token, SiLU, L2 norms, gates; then, per value row i of each state (field guide §02):
//   S' = alpha S;  r_k = S' k;  e = beta (v_i - r_k);  S'' = S' + e k^T;  y_i = S'' q
// using y_i = alpha (S q)_i + e (k . q), so each 512-byte state row is read once and
// written once.  Dot products are warp-shuffle reductions over the row's 128 entries (four
// per lane).  Last, y is RMS-normalised per value head and gated by SiLU(z).
//
// With `slots`, sequence n's state and conv history live in pool slot slots[n] (a resident
// state pool, as a serving loop keeps one); a negative slot marks a padding entry that reads
// and writes nothing, and a slot past the pool sets the device status and skips the entry.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int DEC_ROWS = 8;  // state rows in flight per warp
// Three CTAs (24 warps) per SM: registers capped at 85 per thread, so that more state rows are
// in flight per SM (measured: 194.6 -> 184.1 us per step for 256 sequences; 16 rows per warp at
// two CTAs per SM gave 185.3 us).

template <bool BF16, bool OUT_BF16>
__global__ void __launch_bounds__(256, 3) k_decode(Dims d, const void* __restrict__ q,
                                                const void* __restrict__ k, const void* __restrict__ v,
                                                const void* __restrict__ z, const float* __restrict__ a,
                                                const float* __restrict__ b,
                                                const float* __restrict__ A_log,
                                                const float* __restrict__ dt_bias,
                                                const float* __restrict__ conv_w,
                                                const float* __restrict__ norm_w, void* conv_state,
                                                float* state, void* __restrict__ y,
                                                const int32_t* __restrict__ slots, int n_slots) {
  using E = typename std::conditional<BF16, uint16_t, float>::type;
  const int n = blockIdx.x, j = blockIdx.y;
  int slot = n;
  if (slots) {
    slot = slots[n];
    if (slot < 0) return;  // padding entry
    if (slot >= n_slots) {
      if (threadIdx.x == 0) atomicExch(&g_gdn_status, -8);
      return;
    }
  }
  const int hq = d.h_qk, hv = d.h_v, G = hv / hq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t cconv = (size_t)(2 * hq + hv) * D;
  __shared__ __align__(16) float qs[D];
  __shared__ __align__(16) float ks[D];
  __shared__ __align__(16) float vs[8][D];
  __shared__ __align__(16) float ys[8][D];
  __shared__ float alpha_s[8], beta_s[8];

  // conv + SiLU over this CTA's channels, and the conv-history shift (raw values, bit-exact)
  E* cs = static_cast<E*>(conv_state) + (size_t)slot * 3 * cconv;
  const int nch = 2 * D + G * D;
  for (int c = tid; c < nch; c += blockDim.x) {
    size_t ch;
    E xin;
    float* dst;
    if (c < D) {
      ch = (size_t)j * D + c;
      xin = static_cast<const E*>(q)[((size_t)n * hq + j) * D + c];
      dst = qs + c;
    } else if (c < 2 * D) {
      ch = (size_t)(hq + j) * D + (c - D);
      xin = static_cast<const E*>(k)[((size_t)n * hq + j) * D + (c - D)];
      dst = ks + (c - D);
    } else {
      const int g = (c - 2 * D) / D, cc = (c - 2 * D) % D, hh = j * G + g;
      ch = (size_t)2 * hq * D + (size_t)hh * D + cc;
      xin = static_cast<const E*>(v)[((size_t)n * hv + hh) * D + cc];
      dst = &vs[g][cc];
    }
    const E x0 = cs[ch], x1 = cs[cconv + ch], x2 = cs[2 * cconv + ch];
    const float4 w = *reinterpret_cast<const float4*>(conv_w + ch * 4);
    float f0, f1, f2, f3;
    if constexpr (BF16) {
      f0 = bf2f(x0); f1 = bf2f(x1); f2 = bf2f(x2); f3 = bf2f(xin);
    } else {
      f0 = x0; f1 = x1; f2 = x2; f3 = xin;
    }
    *dst = silu_f(fmaf(w.w, f3, fmaf(w.z, f2, fmaf(w.y, f1, w.x * f0))));
    cs[ch] = x1;
    cs[cconv + ch] = x2;
    cs[2 * cconv + ch] = xin;
  }
  if (tid < G) {
    const int hh = j * G + tid;
    alpha_s[tid] = expf(decay_gate_f(a[(size_t)n * hv + hh], A_log[hh], dt_bias[hh]));
    beta_s[tid] = sigmoid_f(b[(size_t)n * hv + hh]);
  }
  __syncthreads();
  if (warp < 2) {  // L2 norms: warp 0 normalises q (times q_scale), warp 1 normalises k
    float* p = warp ? ks : qs;
    float4 x = *reinterpret_cast<float4*>(p + lane * 4);
    const float ss = warp_sum(x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w);
    const float inv = (warp ? 1.0f : d.q_scale) / sqrtf(ss + d.l2_eps);
    x.x *= inv; x.y *= inv; x.z *= inv; x.w *= inv;
    *reinterpret_cast<float4*>(p + lane * 4) = x;
  }
  __syncthreads();
  const float4 kr = *reinterpret_cast<const float4*>(ks + lane * 4);
  const float4 qr = *reinterpret_cast<const float4*>(qs + lane * 4);
  const float kq = warp_sum(dot4(kr, qr));

  // state rows: G * 128 rows, an equal contiguous share per warp, DEC_ROWS in flight
  const int rows_per_warp = G * D / 8;
  const size_t state0 = ((size_t)slot * hv + (size_t)j * G) * D * D;
  for (int r0 = warp * rows_per_warp; r0 < (warp + 1) * rows_per_warp; r0 += DEC_ROWS) {
    float4 s[DEC_ROWS];
#pragma unroll
    for (int u = 0; u < DEC_ROWS; ++u)
      s[u] = __ldcs(reinterpret_cast<const float4*>(state + state0 + (size_t)(r0 + u) * D + lane * 4));
#pragma unroll
    for (int u = 0; u < DEC_ROWS; ++u) {
      const int row = r0 + u, g = row / D, i = row % D;
      const float rk = warp_sum(dot4(s[u], kr));
      const float rq = warp_sum(dot4(s[u], qr));
      const float al = alpha_s[g];
      const float e = beta_s[g] * (vs[g][i] - al * rk);
      float4 o;
      o.x = fmaf(al, s[u].x, e * kr.x);
      o.y = fmaf(al, s[u].y, e * kr.y);
      o.z = fmaf(al, s[u].z, e * kr.z);
      o.w = fmaf(al, s[u].w, e * kr.w);
      __stcs(reinterpret_cast<float4*>(state + state0 + (size_t)row * D + lane * 4), o);
      if (lane == 0) ys[g][i] = fmaf(al, rq, e * kq);
    }
  }
  __syncthreads();
  for (int g = warp; g < G; g += 8) {
    const float4 yv = *reinterpret_cast<const float4*>(&ys[g][lane * 4]);
    const float ss = warp_sum(yv.x * yv.x + yv.y * yv.y + yv.z * yv.z + yv.w * yv.w);
    const float inv = 1.0f / sqrtf(ss * (1.0f / D) + d.rms_eps);
    const size_t off = ((size_t)n * hv + (size_t)j * G + g) * D + lane * 4;
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

// The decode step's conv history after a prefill: the raw (pre-conv) q | k | v channels of
// each sequence's last three tokens, row r = token te - 3 + r, in the conv_state layout
// [N][3][C_conv].  Rows before the sequence's first token are zeros, as the prefill's own
// history starts at zero.  One CTA per (sequence, row); 16-byte copies.  A cu_seqlens entry
// outside [0, T_tot] or decreasing sets the device status and writes zeros.
template <typename E>
__global__ void __launch_bounds__(256) k_conv_state_out(Dims d, const E* __restrict__ q, const E* __restrict__ k,
                                                        const E* __restrict__ v, const int* __restrict__ cu,
                                                        E* __restrict__ out) {
  const int n = blockIdx.x, r = blockIdx.y;
  int ts = cu ? cu[n] : 0, te = cu ? cu[n + 1] : d.total_tokens;
  if (ts < 0 || te < ts || te > d.total_tokens) {
    if (threadIdx.x == 0) atomicExch(&g_gdn_status, -8);
    ts = te = 0;
  }
  const int t = te - 3 + r;
  const size_t cq = (size_t)d.h_qk * D, cv = (size_t)d.h_v * D, cconv = 2 * cq + cv;
  constexpr int V = 16 / sizeof(E);  // elements per 16-byte copy (never straddles a stream)
  uint4* o = reinterpret_cast<uint4*>(out + ((size_t)n * 3 + r) * cconv);
  for (size_t c = (size_t)threadIdx.x * V; c < cconv; c += (size_t)blockDim.x * V) {
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (t >= ts) {
      const E* src = c < cq ? q + (size_t)t * cq + c
                   : c < 2 * cq ? k + (size_t)t * cq + (c - cq)
                                : v + (size_t)t * cv + (c - 2 * cq);
      x = *reinterpret_cast<const uint4*>(src);
    }
    o[c / V] = x;
  }
}

}  // namespace gdn
