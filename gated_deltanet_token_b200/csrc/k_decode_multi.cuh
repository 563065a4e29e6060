// k_decode_multi.cuh -- K decode tokens per sequence in one pass over the state (K <= 8).
//
// Same per-token rule as k_decode (field guide §02, steps 1-6, then the gated RMSNorm), applied
// to K consecutive tokens of each sequence.  The state rows stay in registers across the K
// tokens, so each 512-byte row is read once and written once per call instead of once per
// token.  Conv: the K new raw rows follow the three history rows; the history keeps the last
// three raw rows.  One CTA per (sequence n, QK head j) as in k_decode.
//
// Row layout: eight lanes share a state row, each holding four groups of four columns
// (columns 32 c + 4 (lane % 8) .. + 3, c = 0..3).  A warp works on four rows at once, and the
// two dot products of a token (S'k and S'q) reduce over eight lanes in three shuffle levels --
// for four rows together.  A warp takes its rows in groups of four (one four-row slab): each
// group is copied into shared memory by asynchronous 16-byte copies two groups ahead (double-
// buffered; the first two start before the conv prologue), so the next 2 KB of state is in
// flight while the current group is updated in registers; the updated rows go straight back
// to global memory.  The dot products and the row update use paired fp32 FMAs, and the token
// loop runs two tokens at a time.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int DECM_KMAX = 8;
constexpr int DECM_LPR = 8;             // lanes per state row
constexpr int DECM_CPL = D / DECM_LPR;  // columns per lane: 16
constexpr int DECM_SLABS = 1;           // four-row slabs per group

constexpr int DECM_WARPS = 8;
constexpr int DECM_GROUP = 4 * DECM_SLABS;                      // state rows per group
constexpr int DECM_BUF_FLOATS = 2 * DECM_WARPS * DECM_GROUP * D;  // two group buffers per warp

// Dynamic shared memory of one CTA (floats): the state-row buffers; q, k [K][D]; v, y [K][G][D];
// alpha, beta [K][G]; k . q [K].
__host__ __device__ constexpr size_t decm_smem_bytes(int K, int G) {
  return (size_t)(DECM_BUF_FLOATS + 2 * K * D + 2 * K * G * D + 2 * K * G + K) * sizeof(float);
}
constexpr size_t DECM_SMEM = decm_smem_bytes(DECM_KMAX, 8);

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
  if (K < 1 || K > DECM_KMAX || G > 8) {
    if (tid == 0) atomicExch(&g_gdn_status, -6);
    return;
  }
  extern __shared__ __align__(16) float dm[];
  float* sbuf = dm;               // [warps][2][8 rows][D] state-row buffers
  float* qs = sbuf + DECM_BUF_FLOATS;  // [K][D]
  float* ks = qs + K * D;         // [K][D]
  float* vs = ks + K * D;         // [K][G][D]
  float* ys = vs + K * G * D;     // [K][G][D]
  float* al = ys + K * G * D;     // [K][G]  e^{g}
  float* be = al + K * G;         // [K][G]  beta
  float* kqv = be + K * G;        // [K]     k_t . q_t

  const int sub = lane >> 3, cl = (lane & 7) * 4;
  const int rows_per_warp = G * D / DECM_WARPS;  // a multiple of DECM_GROUP
  const int ngroups = rows_per_warp / DECM_GROUP;
  const size_t wrow0 = ((size_t)n * hv + (size_t)j * G) * D + (size_t)warp * rows_per_warp;  // first row
  float* wbuf = sbuf + warp * 2 * DECM_GROUP * D;
  // group gi of this warp's rows into buffer gi & 1: 128 chunks of 16 bytes, 4 per lane
  auto load_group = [&](int gi) {
    const float* src = state + (wrow0 + (size_t)gi * DECM_GROUP) * D;
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(wbuf + (gi & 1) * DECM_GROUP * D));
#pragma unroll
    for (int m = 0; m < DECM_GROUP * D / 4 / 32; ++m) {
      const int idx = lane + 32 * m;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + idx * 16), "l"(src + idx * 4) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // the first two groups start streaming now, under the conv, gates and norms below
  load_group(0);
  if (ngroups > 1) load_group(1);
  else asm volatile("cp.async.commit_group;" ::: "memory");
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
      dstride = G * D;
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
    al[i] = expf(decay_gate_f(a[o], A_log[hh], dt_bias[hh]));
    be[i] = sigmoid_f(b[o]);
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

  // State rows: an equal contiguous share of the CTA's G * 128 rows per warp (a multiple of 16),
  // DECM_SLABS four-row slabs at a time.  Lane: row sub = lane / 8 of a slab, columns
  // 32 c4 + cl .. + 3 for c4 = 0..3.  Per token, for each row i of value head g:
  //   S' = alpha S;  r_k = S' k;  e = beta (v_i - r_k);  S'' = S' + e k^T;  y_i = S'' q
  // with y_i = alpha (S q) + e (k . q).
  for (int gi = 0; gi < ngroups; ++gi) {
    // committed so far: groups 0 .. gi + 1 (an empty group stands in past the last one)
    asm volatile("cp.async.wait_group 1;" ::: "memory");  // this lane's copies of group gi landed
    __syncwarp();                                           // ... and every lane's
    const float* gb = wbuf + (gi & 1) * DECM_GROUP * D;
    float4 s[DECM_SLABS][DECM_CPL / 4];
#pragma unroll
    for (int sl = 0; sl < DECM_SLABS; ++sl)
#pragma unroll
      for (int c4 = 0; c4 < DECM_CPL / 4; ++c4)
        s[sl][c4] = *reinterpret_cast<const float4*>(gb + (4 * sl + sub) * D + 32 * c4 + cl);
    __syncwarp();  // every lane has read the buffer before group gi + 2 refills it
    if (gi + 2 < ngroups) load_group(gi + 2);
    else asm volatile("cp.async.commit_group;" ::: "memory");
#pragma unroll 2  // two tokens at a time: the second token's k, q loads overlap the first's chain
    for (int t = 0; t < K; ++t) {
      float4 kr[DECM_CPL / 4], qr[DECM_CPL / 4];
#pragma unroll
      for (int c4 = 0; c4 < DECM_CPL / 4; ++c4) {
        kr[c4] = *reinterpret_cast<const float4*>(ks + t * D + 32 * c4 + cl);
        qr[c4] = *reinterpret_cast<const float4*>(qs + t * D + 32 * c4 + cl);
      }
      const float kq = kqv[t];
#pragma unroll
      for (int sl = 0; sl < DECM_SLABS; ++sl) {
        float2 rk2 = make_float2(0.0f, 0.0f), rq2 = rk2;
#pragma unroll
        for (int c4 = 0; c4 < DECM_CPL / 4; ++c4) {
          const float2 s0 = make_float2(s[sl][c4].x, s[sl][c4].y), s1 = make_float2(s[sl][c4].z, s[sl][c4].w);
          rk2 = __ffma2_rn(s0, make_float2(kr[c4].x, kr[c4].y), rk2);
          rk2 = __ffma2_rn(s1, make_float2(kr[c4].z, kr[c4].w), rk2);
          rq2 = __ffma2_rn(s0, make_float2(qr[c4].x, qr[c4].y), rq2);
          rq2 = __ffma2_rn(s1, make_float2(qr[c4].z, qr[c4].w), rq2);
        }
        float rk = rk2.x + rk2.y, rq = rq2.x + rq2.y;
#pragma unroll
        for (int o = 1; o < DECM_LPR; o <<= 1) {  // the eight lanes of the row
          rk += __shfl_xor_sync(0xffffffffu, rk, o);
          rq += __shfl_xor_sync(0xffffffffu, rq, o);
        }
        const int row = warp * rows_per_warp + gi * DECM_GROUP + 4 * sl + sub, g = row / D, i = row % D;
        const float a_ = al[t * G + g];
        const float e = be[t * G + g] * (vs[(t * G + g) * D + i] - a_ * rk);
        const float2 a2 = make_float2(a_, a_), e2 = make_float2(e, e);
#pragma unroll
        for (int c4 = 0; c4 < DECM_CPL / 4; ++c4) {
          const float2 lo = __ffma2_rn(a2, make_float2(s[sl][c4].x, s[sl][c4].y),
                                       __fmul2_rn(e2, make_float2(kr[c4].x, kr[c4].y)));
          const float2 hi = __ffma2_rn(a2, make_float2(s[sl][c4].z, s[sl][c4].w),
                                       __fmul2_rn(e2, make_float2(kr[c4].z, kr[c4].w)));
          s[sl][c4] = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
        if ((lane & (DECM_LPR - 1)) == 0) ys[(t * G + g) * D + i] = fmaf(a_, rq, e * kq);
      }
    }
#pragma unroll
    for (int sl = 0; sl < DECM_SLABS; ++sl) {
      float4* dst = reinterpret_cast<float4*>(state + (wrow0 + (size_t)gi * DECM_GROUP + 4 * sl + sub) * D + cl);
#pragma unroll
      for (int c4 = 0; c4 < DECM_CPL / 4; ++c4) __stcs(dst + 8 * c4, s[sl][c4]);
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  for (int i = warp; i < K * G; i += 8) {  // gated RMSNorm of each (token, value head)
    const int t = i / G, g = i % G;
    const float4 yv = *reinterpret_cast<const float4*>(ys + (t * G + g) * D + lane * 4);
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

}  // namespace gdn
