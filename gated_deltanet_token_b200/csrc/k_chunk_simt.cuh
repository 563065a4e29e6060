// k_chunk_simt.cuh -- chunked gated-delta-rule prefill on CUDA cores, all fp32 (FFMA).
//
// The chunk algebra (an exact rewrite of the per-token rule of the "Qwen3-Next 80B-A3B"
// field guide, §02, steps 1-6), for one chunk of L <= 64 tokens of one value head with
// state S_0 (d_v x d_k) at its start, rows t, s indexing the chunk's tokens:
//   gamma_t = sum_{r<=t} g_r                                    (chunk-local decay prefix)
//   A[t][s] = beta_t e^{gamma_t - gamma_s} (k_t . k_s), s < t   (strictly lower triangular)
//   W  = (I + A)^-1 diag(beta e^gamma) K,   U' = (I + A)^-1 diag(beta) V
//   U  = U' - W S_0^T                                            (the delta-rule errors)
//   Y  = diag(e^gamma) Q S_0^T + (M o Q K^T) U,  M[t][s] = e^{gamma_t - gamma_s}, s <= t
//   S_L = e^{gamma_L} S_0 + U^T diag(e^{gamma_L - gamma}) K
// The last line is the chunk-loop state update of the "Qwen3.8-Flash-Next" model notes
// (state * chunk decay + key^T @ new values), in the column-vector convention.
//
// Phase A (parallel over chunks x value heads) computes gamma, M o QK^T, W and U'.
// Phase B (sequential over one sequence's chunks, parallel over value heads and 32-row
// slices of the state: value rows of S evolve independently) computes U, Y and S.
// Decay factors are formed as exp(gamma_t - gamma_s) after masking s <= t, never as a
// ratio, so nothing overflows.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int PA_LD = 132;  // padded row pitch (floats) of 64 x 128 tiles
constexpr int PA_ALD = 68;  // padded row pitch of the 64 x 64 A tile
constexpr size_t PA_SMEM = (size_t)(2 * 64 * PA_LD + 64 * PA_ALD + 4 * 64) * sizeof(float);

// Phase A: grid (chunk, value head), 256 threads.
__global__ void __launch_bounds__(256, 2)
    k_phaseA_simt(Dims d, const ChunkEntry* __restrict__ tab, const float* __restrict__ qn,
                  const float* __restrict__ kn, const float* __restrict__ vc,
                  const float* __restrict__ g, const float* __restrict__ beta,
                  double* __restrict__ gam_out, float* __restrict__ W_out,
                  float* __restrict__ Up_out, float* __restrict__ mqk_out) {
  const ChunkEntry e = tab[blockIdx.x];
  if (e.len == 0) return;
  const int h = blockIdx.y, hq = d.h_qk, hv = d.h_v, j = h / (hv / hq), L = e.len;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ float4 smem_f4[];
  float* Ks = reinterpret_cast<float*>(smem_f4);
  float* Qs = Ks + 64 * PA_LD;
  float* As = Qs + 64 * PA_LD;
  double* gs = reinterpret_cast<double*>(As + 64 * PA_ALD);  // gamma (fp64: see below)
  float* bs = reinterpret_cast<float*>(gs + 64);               // beta
  float* be = bs + 64;                                         // beta * e^gamma

  for (int idx = tid; idx < 64 * 32; idx += 256) {
    const int t = idx >> 5, c4 = (idx & 31) * 4;
    float4 kv = make_float4(0, 0, 0, 0), qv = kv;
    if (t < L) {
      const size_t off = ((size_t)(e.t0 + t) * hq + j) * D + c4;
      kv = *reinterpret_cast<const float4*>(kn + off);
      qv = *reinterpret_cast<const float4*>(qn + off);
    }
    *reinterpret_cast<float4*>(Ks + t * PA_LD + c4) = kv;
    *reinterpret_cast<float4*>(Qs + t * PA_LD + c4) = qv;
  }
  // Inclusive prefix sum of g over the chunk, two tokens per lane, in fp64: every decay
  // factor e^{gamma_t - gamma_s} is formed from a difference of two prefixes, which in fp32
  // would carry an absolute error of ulp(|gamma|) -- about 2e-4 once a few strong decays (g of
  // several hundred) have accumulated in the chunk.
  if (warp == 0) {
    double s0 = lane < L ? g[(size_t)(e.t0 + lane) * hv + h] : 0.0f;
    double s1 = lane + 32 < L ? g[(size_t)(e.t0 + lane + 32) * hv + h] : 0.0f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y0 = __shfl_up_sync(0xffffffffu, s0, o);
      const double y1 = __shfl_up_sync(0xffffffffu, s1, o);
      if (lane >= o) { s0 += y0; s1 += y1; }
    }
    s1 += __shfl_sync(0xffffffffu, s0, 31);
    const float b0 = lane < L ? beta[(size_t)(e.t0 + lane) * hv + h] : 0.0f;
    const float b1 = lane + 32 < L ? beta[(size_t)(e.t0 + lane + 32) * hv + h] : 0.0f;
    gs[lane] = s0; gs[lane + 32] = s1;
    bs[lane] = b0; bs[lane + 32] = b1;
    be[lane] = b0 * expf((float)s0); be[lane + 32] = b1 * expf((float)s1);
    if (lane < L) gam_out[(size_t)(e.t0 + lane) * hv + h] = s0;
    if (lane + 32 < L) gam_out[(size_t)(e.t0 + lane + 32) * hv + h] = s1;
  }
  __syncthreads();

  // K K^T and Q K^T: thread (tb, sb) owns rows tb + 16 r and columns sb + 16 c.
  {
    const int tb = tid >> 4, sb = tid & 15;
    float kk[4][4], qk[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) kk[r][c] = qk[r][c] = 0.0f;
#pragma unroll 4
    for (int jj = 0; jj < D; jj += 4) {
      float4 kt[4], qt[4], ks[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        kt[r] = *reinterpret_cast<const float4*>(Ks + (tb + 16 * r) * PA_LD + jj);
        qt[r] = *reinterpret_cast<const float4*>(Qs + (tb + 16 * r) * PA_LD + jj);
        ks[r] = *reinterpret_cast<const float4*>(Ks + (sb + 16 * r) * PA_LD + jj);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          kk[r][c] += dot4(kt[r], ks[c]);
          qk[r][c] += dot4(qt[r], ks[c]);
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int t = tb + 16 * r, s = sb + 16 * c;
        const float dec = s <= t ? expf((float)(gs[t] - gs[s])) : 0.0f;  // mask before exp
        As[t * PA_ALD + s] = s < t ? bs[t] * dec * kk[r][c] : 0.0f;
        if (t < L) mqk_out[((size_t)(e.t0 + t) * hv + h) * CH + s] = (s <= t) ? dec * qk[r][c] : 0.0f;
      }
  }
  __syncthreads();

  // (I + A) X = [diag(beta e^gamma) K | diag(beta) V]: thread c owns column c and runs the
  // forward substitution down it; A is read by broadcast, X stays in registers.
  {
    const bool isK = tid < 128;
    const int col = tid & 127;
    float x[64];
#pragma unroll
    for (int t = 0; t < 64; ++t) {
      float rhs;
      if (isK) rhs = be[t] * Ks[t * PA_LD + col];
      else rhs = t < L ? bs[t] * vc[((size_t)(e.t0 + t) * hv + h) * D + col] : 0.0f;
#pragma unroll
      for (int s = 0; s < t; ++s) rhs = fmaf(-As[t * PA_ALD + s], x[s], rhs);
      x[t] = rhs;
    }
    float* out = isK ? W_out : Up_out;
#pragma unroll
    for (int t = 0; t < 64; ++t)
      if (t < L) out[((size_t)(e.t0 + t) * hv + h) * D + col] = x[t];
  }
}

constexpr int PB_VS = 32;   // value rows of the state per CTA
constexpr int PB_LD = 132;  // row pitch of 128-wide tiles
constexpr int PB_ULD = 36;  // row pitch of the U tile
constexpr int PB_MLD = 68;  // row pitch of the M o QK^T tile
constexpr size_t PB_SMEM =
    (size_t)(PB_VS * PB_LD + 3 * 64 * PB_LD + 64 * PB_ULD + 64 * PB_MLD + 2 * 64) * sizeof(float);

// Phase B: grid (sequence, value head, state slice), 256 threads.
__global__ void __launch_bounds__(256, 1)
    k_phaseB_simt(Dims d, const int* __restrict__ cu, const float* __restrict__ qn,
                  const float* __restrict__ kn, const double* __restrict__ gam,
                  const float* __restrict__ Wg, const float* __restrict__ Upg,
                  const float* __restrict__ mqk, const float* init_state,
                  float* __restrict__ y_raw, float* final_state) {
  const int n = blockIdx.x, h = blockIdx.y, i0 = blockIdx.z * PB_VS;
  const int hq = d.h_qk, hv = d.h_v, j = h / (hv / hq);
  const int tid = threadIdx.x;
  const int ts = cu ? cu[n] : 0, te = cu ? cu[n + 1] : d.total_tokens;
  extern __shared__ float4 smem_f4[];
  float* Ss = reinterpret_cast<float*>(smem_f4);  // [32][PB_LD]  state slice S[i0 + r][:]
  float* Ws = Ss + PB_VS * PB_LD;                  // [64][PB_LD]  W
  float* Qs = Ws + 64 * PB_LD;                     // [64][PB_LD]  Q
  float* Ks = Qs + 64 * PB_LD;                     // [64][PB_LD]  diag(e^{gamma_L - gamma}) K
  float* Us = Ks + 64 * PB_LD;                     // [64][PB_ULD] U' then U (slice columns)
  float* Ms = Us + 64 * PB_ULD;                    // [64][PB_MLD] M o QK^T
  double* gs = reinterpret_cast<double*>(Ms + 64 * PB_MLD);  // [64] gamma (fp64)

  const size_t sbase = (((size_t)n * hv + h) * D + i0) * D;
  for (int idx = tid; idx < PB_VS * 32; idx += 256) {
    const int r = idx >> 5, c4 = (idx & 31) * 4;
    const float4 v = init_state ? *reinterpret_cast<const float4*>(init_state + sbase + (size_t)r * D + c4)
                                : make_float4(0, 0, 0, 0);
    *reinterpret_cast<float4*>(Ss + r * PB_LD + c4) = v;
  }

  for (int t0 = ts; t0 < te; t0 += CH) {
    const int L = min(CH, te - t0);
    __syncthreads();  // the previous chunk is finished with every tile
    if (tid < 64) gs[tid] = tid < L ? gam[(size_t)(t0 + tid) * hv + h] : 0.0;
    __syncthreads();
    const double gL = gs[L - 1];
    for (int idx = tid; idx < 64 * 32; idx += 256) {
      const int t = idx >> 5, c4 = (idx & 31) * 4;
      float4 wv = make_float4(0, 0, 0, 0), qv = wv, kv = wv;
      if (t < L) {
        const size_t tk = ((size_t)(t0 + t) * hq + j) * D + c4;
        wv = *reinterpret_cast<const float4*>(Wg + ((size_t)(t0 + t) * hv + h) * D + c4);
        qv = *reinterpret_cast<const float4*>(qn + tk);
        kv = *reinterpret_cast<const float4*>(kn + tk);
        const float f = expf((float)(gL - gs[t]));
        kv.x *= f; kv.y *= f; kv.z *= f; kv.w *= f;
      }
      *reinterpret_cast<float4*>(Ws + t * PB_LD + c4) = wv;
      *reinterpret_cast<float4*>(Qs + t * PB_LD + c4) = qv;
      *reinterpret_cast<float4*>(Ks + t * PB_LD + c4) = kv;
    }
    for (int idx = tid; idx < 64 * 8; idx += 256) {
      const int t = idx >> 3, c4 = (idx & 7) * 4;
      const float4 uv = t < L ? *reinterpret_cast<const float4*>(Upg + ((size_t)(t0 + t) * hv + h) * D + i0 + c4)
                              : make_float4(0, 0, 0, 0);
      *reinterpret_cast<float4*>(Us + t * PB_ULD + c4) = uv;
    }
    for (int idx = tid; idx < 64 * 16; idx += 256) {
      const int t = idx >> 4, c4 = (idx & 15) * 4;
      const float4 mv = t < L ? *reinterpret_cast<const float4*>(mqk + ((size_t)(t0 + t) * hv + h) * CH + c4)
                              : make_float4(0, 0, 0, 0);
      *reinterpret_cast<float4*>(Ms + t * PB_MLD + c4) = mv;
    }
    __syncthreads();

    // U = U' - W S^T and Q S^T: thread (tb, ib) owns rows tb + 16 r, slice columns ib + 16 c.
    const int tb = tid >> 4, ib = tid & 15;
    float u[4][2], qs[4][2];
    {
      float wa[4][2], qa[4][2];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 2; ++c) wa[r][c] = qa[r][c] = 0.0f;
#pragma unroll 4
      for (int jj = 0; jj < D; jj += 4) {
        float4 wr[4], qr[4], sr[2];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          wr[r] = *reinterpret_cast<const float4*>(Ws + (tb + 16 * r) * PB_LD + jj);
          qr[r] = *reinterpret_cast<const float4*>(Qs + (tb + 16 * r) * PB_LD + jj);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) sr[c] = *reinterpret_cast<const float4*>(Ss + (ib + 16 * c) * PB_LD + jj);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            wa[r][c] += dot4(wr[r], sr[c]);
            qa[r][c] += dot4(qr[r], sr[c]);
          }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = tb + 16 * r;
        const float eg = t < L ? expf((float)gs[t]) : 0.0f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          u[r][c] = Us[t * PB_ULD + ib + 16 * c] - wa[r][c];
          qs[r][c] = eg * qa[r][c];
        }
      }
    }
    __syncthreads();  // every thread has read S and U' before they change
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 2; ++c) Us[(tb + 16 * r) * PB_ULD + ib + 16 * c] = u[r][c];
    __syncthreads();

    // Y = diag(e^gamma) Q S^T + (M o QK^T) U
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int t = tb + 16 * r;
      float y0 = qs[r][0], y1 = qs[r][1];
      for (int s = 0; s <= t; ++s) {
        const float m = Ms[t * PB_MLD + s];
        y0 = fmaf(m, Us[s * PB_ULD + ib], y0);
        y1 = fmaf(m, Us[s * PB_ULD + ib + 16], y1);
      }
      if (t < L) {
        float* yr = y_raw + ((size_t)(t0 + t) * hv + h) * D + i0;
        yr[ib] = y0;
        yr[ib + 16] = y1;
      }
    }

    // S <- e^{gamma_L} S + U^T diag(e^{gamma_L - gamma}) K: thread (rb, jb) owns rows
    // rb + 8 r and columns 4 jb .. 4 jb + 3.
    {
      const int rb = tid >> 5, jb = (tid & 31) * 4;
      const float eL = expf((float)gL);
      float4 acc[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 s0 = *reinterpret_cast<const float4*>(Ss + (rb + 8 * r) * PB_LD + jb);
        acc[r] = make_float4(eL * s0.x, eL * s0.y, eL * s0.z, eL * s0.w);
      }
      for (int s = 0; s < L; ++s) {
        const float4 kv = *reinterpret_cast<const float4*>(Ks + s * PB_LD + jb);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float uu = Us[s * PB_ULD + rb + 8 * r];
          acc[r].x = fmaf(uu, kv.x, acc[r].x);
          acc[r].y = fmaf(uu, kv.y, acc[r].y);
          acc[r].z = fmaf(uu, kv.z, acc[r].z);
          acc[r].w = fmaf(uu, kv.w, acc[r].w);
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) *reinterpret_cast<float4*>(Ss + (rb + 8 * r) * PB_LD + jb) = acc[r];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < PB_VS * 32; idx += 256) {
    const int r = idx >> 5, c4 = (idx & 31) * 4;
    *reinterpret_cast<float4*>(final_state + sbase + (size_t)r * D + c4) =
        *reinterpret_cast<const float4*>(Ss + r * PB_LD + c4);
  }
}

}  // namespace gdn
