// k_bwd.cuh -- backward pass of the gated delta rule's recurrence core (fp32, CUDA cores).
//
// Forward (field guide §02, steps 1-6, column-vector state S of d_v x d_k), alpha_t = e^{g_t}:
//   S'_t = alpha_t S_{t-1};  e_t = v_t - S'_t k_t;  S_t = S'_t + beta_t e_t k_t^T;  y_t = S_t q_t.
// Reverse mode, walking the tokens from the last with D = dL/dS_t (seeded with dL/dS_T):
//   D += dy_t q_t^T;  dq_t = S_t^T dy_t;  w = D k_t;  de_t = beta_t w;  dbeta_t = e_t . w;
//   dv_t = de_t;  dk_t = beta_t D^T e_t - S'_t^T de_t;  dS'_t = D - de_t k_t^T;
//   dg_t = alpha_t <dS'_t, S_{t-1}>;  D <- alpha_t dS'_t;  finally dL/dS_0 = D.
//
// One CTA of 512 threads per (sequence, value head): warp w owns state rows 8w .. 8w + 7, lane
// l columns 4l .. 4l + 3, so a thread keeps 32 elements of S (forward) and of D (reverse) in
// registers.  Row dot products (S' k, D k) are warp reductions; the column sums of dq, dk and the
// scalars dbeta, dg are reduced over the 16 warps through shared memory, double-buffered by
// token parity (one barrier per token).
//   1. Forward over the sequence, storing the state at every chunk start (checkpoints).
//   2. For each chunk from the last: recompute its states from the checkpoint into a scratch
//      that only the storing thread reads back (its own 32 elements per token), then walk the
//      chunk's tokens in reverse.
// dq and dk are written per value head; k_bwd_sum adds the value heads that share a QK head.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int BW_THREADS = 512;
constexpr int BW_ROWS = 8;                             // state rows per warp
constexpr int BW_EL = BW_ROWS * 4;                     // state elements per thread
constexpr size_t BW_STATE_FLOATS = (size_t)D * D;      // one state of a value head
constexpr int BW_RED = 2 * D + 2;                      // dq | dk | dbeta | dalpha partials per warp
constexpr int BW_RED_LD = 2 * D + 4;                   // their row pitch (16-byte aligned rows)

// Floats of one checkpoint (a value head's state, thread-major: [threads][32]) and of one
// CTA's chunk scratch ([64 tokens][threads][32]).
constexpr size_t BW_CK_FLOATS = (size_t)BW_THREADS * BW_EL;
constexpr size_t BW_SCR_FLOATS = (size_t)CH * BW_THREADS * BW_EL;

__device__ __forceinline__ void bw_load(const float* p, float* x) {
#pragma unroll
  for (int i = 0; i < BW_EL / 4; ++i) {
    const float4 f = reinterpret_cast<const float4*>(p)[i];
    x[4 * i] = f.x; x[4 * i + 1] = f.y; x[4 * i + 2] = f.z; x[4 * i + 3] = f.w;
  }
}
__device__ __forceinline__ void bw_store(float* p, const float (&x)[BW_EL]) {
#pragma unroll
  for (int i = 0; i < BW_EL / 4; ++i)
    reinterpret_cast<float4*>(p)[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}

// One forward token on the thread's elements (rows r of BW_ROWS, columns c of 4): S <- S'' with
// e_r = v_r - (alpha S k)_r.  vrow: the warp's BW_ROWS values of v_t.
__device__ __forceinline__ void bw_forward_token(float (&S)[BW_EL], float a, float bt, const float4 k4,
                                                 const float* vrow) {
  const float kc[4] = {k4.x, k4.y, k4.z, k4.w};
  float u[BW_ROWS];
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r) {
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      S[4 * r + c] *= a;
      s = fmaf(S[4 * r + c], kc[c], s);
    }
    u[r] = s;
  }
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r) u[r] = warp_sum(u[r]);
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r) {
    const float e = bt * (__ldg(vrow + r) - u[r]);
#pragma unroll
    for (int c = 0; c < 4; ++c) S[4 * r + c] = fmaf(e, kc[c], S[4 * r + c]);
  }
}

__global__ void __launch_bounds__(BW_THREADS, 1)
    k_bwd(Dims d, const int* __restrict__ cu, const int* __restrict__ seq_chunk0, const float* __restrict__ qh,
          const float* __restrict__ kh,
          const float* __restrict__ v, const float* __restrict__ g, const float* __restrict__ beta,
          const float* __restrict__ init_state, const float* __restrict__ dy, const float* __restrict__ dS_final,
          float* __restrict__ dv, float* __restrict__ dg, float* __restrict__ dbeta, float* __restrict__ dS_init,
          float* __restrict__ ck_ws, float* __restrict__ scr_ws, float* __restrict__ dqh, float* __restrict__ dkh) {
  const int n = blockIdx.x, h = blockIdx.y;
  const int hq = d.h_qk, hv = d.h_v, G = hv / hq, j = h / G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ts = cu ? cu[n] : 0, te = cu ? cu[n + 1] : d.total_tokens;
  const int nchunks = te > ts ? (te - ts + CH - 1) / CH : 0;
  __shared__ __align__(16) float red[2][BW_THREADS / 32][BW_RED_LD];
  const size_t cta = (size_t)n * hv + h;
  const int gc0 = seq_chunk0 ? seq_chunk0[n] : 0;  // the sequence's first chunk slot
  // checkpoint of chunk ci of this (sequence, value head): slot (gc0 + ci, h)
  auto ckp = [&](int ci) { return ck_ws + ((size_t)(gc0 + ci) * hv + h) * BW_CK_FLOATS + (size_t)tid * BW_EL; };
  float* scr = scr_ws + cta * BW_SCR_FLOATS;
  const size_t sbase = cta * BW_STATE_FLOATS;
  const int r0 = warp * BW_ROWS, c0 = lane * 4;  // rows r0 .. r0 + 7, columns c0 .. c0 + 3
  auto elem = [&](int r, int c) { return (size_t)(r0 + r) * D + c0 + c; };

  // ---- 1. forward, a checkpoint at every chunk start ---------------------------------------
  float S[BW_EL];
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) S[4 * r + c] = init_state ? init_state[sbase + elem(r, c)] : 0.0f;
  for (int ci = 0; ci < nchunks; ++ci) {
    bw_store(ckp(ci), S);
    const int t0 = ts + ci * CH, L = min(CH, te - t0);
    for (int tt = 0; tt < L; ++tt) {
      const int t = t0 + tt;
      const float4 k4 = *reinterpret_cast<const float4*>(kh + ((size_t)t * hq + j) * D + c0);
      bw_forward_token(S, __expf(g[(size_t)t * hv + h]), beta[(size_t)t * hv + h], k4,
                       v + ((size_t)t * hv + h) * D + r0);
    }
  }

  // ---- 2. reverse, chunk by chunk from the last ---------------------------------------------
  float Dm[BW_EL];
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) Dm[4 * r + c] = dS_final ? dS_final[sbase + elem(r, c)] : 0.0f;
  int par = 0;
  for (int ci = nchunks - 1; ci >= 0; --ci) {
    const int t0 = ts + ci * CH, L = min(CH, te - t0);
    // recompute the chunk's states S_{t-1} (before each token) into this thread's scratch
    bw_load(ckp(ci), S);
    for (int tt = 0; tt < L; ++tt) {
      const int t = t0 + tt;
      bw_store(scr + ((size_t)tt * BW_THREADS + tid) * BW_EL, S);
      const float4 k4 = *reinterpret_cast<const float4*>(kh + ((size_t)t * hq + j) * D + c0);
      bw_forward_token(S, __expf(g[(size_t)t * hv + h]), beta[(size_t)t * hv + h], k4,
                       v + ((size_t)t * hv + h) * D + r0);
    }
    for (int tt = L - 1; tt >= 0; --tt) {
      const int t = t0 + tt;
      float* Sprev = S;  // S_{t-1}: this thread's elements, from its scratch
      bw_load(scr + ((size_t)tt * BW_THREADS + tid) * BW_EL, Sprev);
      const float a = __expf(g[(size_t)t * hv + h]), bt = beta[(size_t)t * hv + h];
      const float4 k4 = *reinterpret_cast<const float4*>(kh + ((size_t)t * hq + j) * D + c0);
      const float4 q4 = *reinterpret_cast<const float4*>(qh + ((size_t)t * hq + j) * D + c0);
      const float* vrow = v + ((size_t)t * hv + h) * D + r0;
      const float* yrow = dy + ((size_t)t * hv + h) * D + r0;
      const float kc[4] = {k4.x, k4.y, k4.z, k4.w}, qc[4] = {q4.x, q4.y, q4.z, q4.w};
      // e_t = v_t - S'_t k_t with S'_t = alpha S_{t-1}
      float e[BW_ROWS];
#pragma unroll
      for (int r = 0; r < BW_ROWS; ++r) {
        float s = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) s = fmaf(Sprev[4 * r + c], kc[c], s);
        e[r] = s;
      }
#pragma unroll
      for (int r = 0; r < BW_ROWS; ++r) e[r] = __ldg(vrow + r) - a * warp_sum(e[r]);
      // dq partial: S_t^T dy (S_t = alpha S_{t-1} + beta e k^T);  D += dy q^T;  w = D k
      float dqp[4] = {0.0f, 0.0f, 0.0f, 0.0f}, w[BW_ROWS];
#pragma unroll
      for (int r = 0; r < BW_ROWS; ++r) {
        const float gy = __ldg(yrow + r);
        float s = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          dqp[c] = fmaf(gy, fmaf(a, Sprev[4 * r + c], bt * e[r] * kc[c]), dqp[c]);
          Dm[4 * r + c] = fmaf(gy, qc[c], Dm[4 * r + c]);
          s = fmaf(Dm[4 * r + c], kc[c], s);
        }
        w[r] = s;
      }
#pragma unroll
      for (int r = 0; r < BW_ROWS; ++r) w[r] = warp_sum(w[r]);
      // de = beta w (= dv);  dbeta = e . w;  dk partial = beta D^T e - S'^T de;
      // dS' = D - de k^T;  dalpha partial = <dS', S_{t-1}>;  D <- alpha dS'
      float dkp[4] = {0.0f, 0.0f, 0.0f, 0.0f}, dbp = 0.0f, dap = 0.0f;
#pragma unroll
      for (int r = 0; r < BW_ROWS; ++r) {
        const float de = bt * w[r];
        dbp = fmaf(e[r], w[r], dbp);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          dkp[c] = fmaf(bt * e[r], Dm[4 * r + c], fmaf(-de * a, Sprev[4 * r + c], dkp[c]));
          const float dsp = fmaf(-de, kc[c], Dm[4 * r + c]);
          dap = fmaf(dsp, Sprev[4 * r + c], dap);
          Dm[4 * r + c] = a * dsp;
        }
        if (lane == r) dv[((size_t)t * hv + h) * D + r0 + r] = de;
      }
      dap = warp_sum(dap);
      float* rw = red[par][warp];
      *reinterpret_cast<float4*>(rw + c0) = make_float4(dqp[0], dqp[1], dqp[2], dqp[3]);
      *reinterpret_cast<float4*>(rw + D + c0) = make_float4(dkp[0], dkp[1], dkp[2], dkp[3]);
      if (lane == 0) {
        rw[2 * D] = dbp;
        rw[2 * D + 1] = dap;
      }
      __syncthreads();
      if (tid < BW_RED) {  // sums over the warps, in warp order
        float s2 = 0.0f;
#pragma unroll 8
        for (int ww = 0; ww < BW_THREADS / 32; ++ww) s2 += red[par][ww][tid];
        if (tid < D) dqh[((size_t)t * hv + h) * D + tid] = s2;
        else if (tid < 2 * D) dkh[((size_t)t * hv + h) * D + tid - D] = s2;
        else if (tid == 2 * D) dbeta[(size_t)t * hv + h] = s2;
        else dg[(size_t)t * hv + h] = a * s2;
      }
      par ^= 1;  // the next token writes the other buffer; this one is read before the next barrier
    }
  }
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) dS_init[sbase + elem(r, c)] = Dm[4 * r + c];
}

// dq, dk of QK head j = the sum over its value heads, in head order.
__global__ void __launch_bounds__(128) k_bwd_sum(Dims d, const float* __restrict__ dqh, const float* __restrict__ dkh,
                                                 float* __restrict__ dq, float* __restrict__ dk) {
  const int t = blockIdx.x, j = blockIdx.y, c = threadIdx.x;
  const int hq = d.h_qk, hv = d.h_v, G = hv / hq;
  float sq = 0.0f, sk = 0.0f;
  for (int gg = 0; gg < G; ++gg) {
    const size_t o = ((size_t)t * hv + j * G + gg) * D + c;
    sq += dqh[o];
    sk += dkh[o];
  }
  dq[((size_t)t * hq + j) * D + c] = sq;
  dk[((size_t)t * hq + j) * D + c] = sk;
}

}  // namespace gdn
