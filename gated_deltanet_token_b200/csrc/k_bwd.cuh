// k_bwd.cuh -- backward pass of the gated delta rule's recurrence core (fp32, CUDA cores).
//
// Forward (field guide §02, steps 1-6, column-vector state S of d_v x d_k), alpha_t = e^{g_t}:
//   S'_t = alpha_t S_{t-1};  e_t = v_t - S'_t k_t;  S_t = S'_t + beta_t e_t k_t^T;  y_t = S_t q_t.
// Reverse mode, walking the tokens from the last with D = dL/dS_t (seeded with dL/dS_T):
//   D += dy_t q_t^T;  dq_t = S_t^T dy_t;  w = D k_t;  de_t = beta_t w;  dbeta_t = e_t . w;
//   dv_t = de_t;  dk_t = beta_t D^T e_t - S'_t^T de_t;  dS'_t = D - de_t k_t^T;
//   dg_t = alpha_t <dS'_t, S_{t-1}>;  D <- alpha_t dS'_t;  finally dL/dS_0 = D.
//
// Rows of S (value components) evolve independently in both directions; only dq, dk, dbeta and
// dg sum over rows.  So one CTA of 256 threads serves one (sequence, value head, slice of 32
// rows): warp w owns slice rows 4w .. 4w + 3, lane l columns 4l .. 4l + 3, 16 elements of S
// (forward) and of D (reverse) per thread.  Row dot products (S' k, D k) are warp reductions;
// the column sums of dq, dk and the scalars dbeta, dg are reduced over the 8 warps through
// shared memory (double-buffered by token parity, one barrier per token) and written per slice;
// k_bwd_sum adds the slices and the value heads that share a QK head, in a fixed order.
//   1. Forward over the sequence, storing the state at every 64-token chunk start (global).
//   2. For each chunk from the last: its inputs go to shared memory; a forward pass over the
//      chunk keeps the state at every 8th token in shared memory; then, per 8-token sub-chunk
//      from the last, the 8 states before its tokens are recomputed into registers and the
//      sub-chunk's tokens are walked in reverse.  No state sequence goes through global memory.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

constexpr int BW_SL = 4;                               // row slices (CTAs) per value head
constexpr int BW_NR = D / BW_SL;                       // 32 state rows per CTA
constexpr int BW_THREADS = 256;
constexpr int BW_WARPS = BW_THREADS / 32;
constexpr int BW_ROWS = BW_NR / BW_WARPS;              // 4 state rows per warp
constexpr int BW_EL = BW_ROWS * 4;                     // 16 state elements per thread
constexpr int BW_SUB = 8;                              // tokens per sub-chunk
constexpr int BW_NSUB = CH / BW_SUB;                   // sub-chunks per chunk
constexpr int BW_RED = 2 * D + 2;                      // dq | dk | dbeta | dalpha partials
constexpr int BW_RED_LD = 2 * D + 4;                   // their row pitch (16-byte aligned rows)
constexpr size_t BW_CK_FLOATS = (size_t)D * D;         // one checkpoint of a value head's state

// Shared memory, in floats: the chunk's k, q (64 x 128), v and dy of the slice (64 x 32),
// alpha and beta (64); the sub-chunk checkpoints ([8][4 quads][256 threads] float4, so that a
// warp's accesses are consecutive); the per-warp partials [2][8][BW_RED_LD].
constexpr int BWS_K = 0, BWS_Q = BWS_K + CH * D, BWS_V = BWS_Q + CH * D, BWS_DY = BWS_V + CH * BW_NR;
constexpr int BWS_A = BWS_DY + CH * BW_NR, BWS_B = BWS_A + CH, BWS_SUBCK = BWS_B + CH;
constexpr int BWS_RED = BWS_SUBCK + BW_NSUB * BW_EL * BW_THREADS;
constexpr size_t BW_SMEM = (size_t)(BWS_RED + 2 * BW_WARPS * BW_RED_LD) * 4;
static_assert(BW_SMEM <= 227 * 1024, "k_bwd shared memory");

// One forward token on the thread's elements (rows r of BW_ROWS, columns c of 4): S <- S'' with
// e_r = v_r - (alpha S k)_r.  k4: the thread's 4 key components; vrow: the warp's BW_ROWS values.
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
    const float e = bt * (vrow[r] - u[r]);
#pragma unroll
    for (int c = 0; c < 4; ++c) S[4 * r + c] = fmaf(e, kc[c], S[4 * r + c]);
  }
}

__global__ void __launch_bounds__(BW_THREADS, 1)
    k_bwd(Dims d, const int* __restrict__ cu, const int* __restrict__ seq_chunk0, const float* __restrict__ qh,
          const float* __restrict__ kh, const float* __restrict__ v, const float* __restrict__ g,
          const float* __restrict__ beta, const float* __restrict__ init_state, const float* __restrict__ dy,
          const float* __restrict__ dS_final, float* __restrict__ dv, float* __restrict__ dS_init,
          float* __restrict__ ck_ws, float* __restrict__ part) {
  extern __shared__ __align__(16) float bsm[];
  const int n = blockIdx.x, h = blockIdx.y, sl = blockIdx.z;
  const int hq = d.h_qk, hv = d.h_v, G = hv / hq, j = h / G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ts = cu ? cu[n] : 0, te = cu ? cu[n + 1] : d.total_tokens;
  const int nchunks = te > ts ? (te - ts + CH - 1) / CH : 0;
  const int gc0 = seq_chunk0 ? seq_chunk0[n] : 0;  // the sequence's first chunk slot
  const int i0 = sl * BW_NR;                       // the slice's first state row
  const int r0 = warp * BW_ROWS, c0 = lane * 4;    // slice rows r0 .. r0 + 3, columns c0 .. c0 + 3
  const size_t sbase = ((size_t)n * hv + h) * D * D;
  auto elem = [&](int r, int c) { return (size_t)(i0 + r0 + r) * D + c0 + c; };
  float* sK = bsm + BWS_K;
  float* sQ = bsm + BWS_Q;
  float* sV = bsm + BWS_V;
  float* sDY = bsm + BWS_DY;
  float* sA = bsm + BWS_A;
  float* sB = bsm + BWS_B;
  float4* sSub = reinterpret_cast<float4*>(bsm + BWS_SUBCK);
  float* red = bsm + BWS_RED;
  // checkpoint of chunk ci: slot (gc0 + ci, h), slice sl, [4 quads][256 threads] float4
  auto ckp = [&](int ci) {
    return reinterpret_cast<float4*>(ck_ws + ((size_t)(gc0 + ci) * hv + h) * BW_CK_FLOATS +
                                     (size_t)sl * BW_EL * BW_THREADS) + tid;
  };
  auto put = [&](float4* p, int stride, const float (&x)[BW_EL]) {
#pragma unroll
    for (int i = 0; i < BW_EL / 4; ++i) p[i * stride] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
  };
  auto get = [&](const float4* p, int stride, float (&x)[BW_EL]) {
#pragma unroll
    for (int i = 0; i < BW_EL / 4; ++i) {
      const float4 f = p[i * stride];
      x[4 * i] = f.x; x[4 * i + 1] = f.y; x[4 * i + 2] = f.z; x[4 * i + 3] = f.w;
    }
  };
  // the chunk's inputs to shared memory (k, v, alpha, beta; with q and dy for the reverse pass)
  auto load_chunk = [&](int t0, int L, bool rev) {
    for (int i = tid; i < L * (D / 4); i += BW_THREADS) {
      const int tt = i / (D / 4), c4 = i % (D / 4);
      const size_t o = ((size_t)(t0 + tt) * hq + j) * D;
      reinterpret_cast<float4*>(sK)[i] = __ldg(reinterpret_cast<const float4*>(kh + o) + c4);
      if (rev) reinterpret_cast<float4*>(sQ)[i] = __ldg(reinterpret_cast<const float4*>(qh + o) + c4);
    }
    for (int i = tid; i < L * (BW_NR / 4); i += BW_THREADS) {
      const int tt = i / (BW_NR / 4), c4 = i % (BW_NR / 4);
      const size_t o = ((size_t)(t0 + tt) * hv + h) * D + i0;
      reinterpret_cast<float4*>(sV)[i] = __ldg(reinterpret_cast<const float4*>(v + o) + c4);
      if (rev) reinterpret_cast<float4*>(sDY)[i] = __ldg(reinterpret_cast<const float4*>(dy + o) + c4);
    }
    for (int i = tid; i < L; i += BW_THREADS) {
      sA[i] = __expf(g[(size_t)(t0 + i) * hv + h]);
      sB[i] = beta[(size_t)(t0 + i) * hv + h];
    }
  };
  auto fwd = [&](float (&S)[BW_EL], int tt) {
    bw_forward_token(S, sA[tt], sB[tt], *reinterpret_cast<const float4*>(sK + tt * D + c0), sV + tt * BW_NR + r0);
  };

  // ---- 1. forward, a checkpoint at every chunk start ---------------------------------------
  float S[BW_EL];
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) S[4 * r + c] = init_state ? init_state[sbase + elem(r, c)] : 0.0f;
  for (int ci = 0; ci < nchunks; ++ci) {
    const int t0 = ts + ci * CH, L = min(CH, te - t0);
    put(ckp(ci), BW_THREADS, S);
    __syncthreads();  // the previous chunk's inputs are no longer read
    load_chunk(t0, L, false);
    __syncthreads();
    for (int tt = 0; tt < L; ++tt) fwd(S, tt);
  }

  // ---- 2. reverse, chunk by chunk from the last ---------------------------------------------
  float Dm[BW_EL];
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) Dm[4 * r + c] = dS_final ? dS_final[sbase + elem(r, c)] : 0.0f;
  int par = 0;
  const size_t T = (size_t)d.total_tokens;
  for (int ci = nchunks - 1; ci >= 0; --ci) {
    const int t0 = ts + ci * CH, L = min(CH, te - t0);
    __syncthreads();  // the later chunk's inputs and partials are no longer read
    load_chunk(t0, L, true);
    get(ckp(ci), BW_THREADS, S);
    __syncthreads();
    // the state before every 8th token, to this thread's own sub-checkpoint slots
    for (int tt = 0; tt < L; ++tt) {
      if (tt % BW_SUB == 0) put(sSub + (tt / BW_SUB) * BW_EL / 4 * BW_THREADS + tid, BW_THREADS, S);
      fwd(S, tt);
    }
    for (int sc = (L + BW_SUB - 1) / BW_SUB - 1; sc >= 0; --sc) {
      const int tb = sc * BW_SUB, nt = min(BW_SUB, L - tb);  // block-uniform
      float St[BW_SUB][BW_EL];  // St[i]: the state before token tb + i
      get(sSub + sc * BW_EL / 4 * BW_THREADS + tid, BW_THREADS, St[0]);
#pragma unroll
      for (int i = 1; i < BW_SUB; ++i) {
        if (i < nt) {
#pragma unroll
          for (int x = 0; x < BW_EL; ++x) St[i][x] = St[i - 1][x];
          fwd(St[i], tb + i - 1);
        }
      }
#pragma unroll
      for (int i = BW_SUB - 1; i >= 0; --i) {
        if (i >= nt) continue;
        const int tt = tb + i, t = t0 + tt;
        const float* Sprev = St[i];
        const float a = sA[tt], bt = sB[tt];
        const float4 k4 = *reinterpret_cast<const float4*>(sK + tt * D + c0);
        const float4 q4 = *reinterpret_cast<const float4*>(sQ + tt * D + c0);
        const float* vrow = sV + tt * BW_NR + r0;
        const float* yrow = sDY + tt * BW_NR + r0;
        const float kc[4] = {k4.x, k4.y, k4.z, k4.w}, qc[4] = {q4.x, q4.y, q4.z, q4.w};
        // e_t = v_t - S'_t k_t with S'_t = alpha S_{t-1}
        float e[BW_ROWS];
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) {
          float s2 = 0.0f;
#pragma unroll
          for (int c = 0; c < 4; ++c) s2 = fmaf(Sprev[4 * r + c], kc[c], s2);
          e[r] = s2;
        }
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) e[r] = vrow[r] - a * warp_sum(e[r]);
        // dq partial: S_t^T dy (S_t = alpha S_{t-1} + beta e k^T);  D += dy q^T;  w = D k
        float dqp[4] = {0.0f, 0.0f, 0.0f, 0.0f}, w[BW_ROWS];
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) {
          const float gy = yrow[r];
          float s2 = 0.0f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            dqp[c] = fmaf(gy, fmaf(a, Sprev[4 * r + c], bt * e[r] * kc[c]), dqp[c]);
            Dm[4 * r + c] = fmaf(gy, qc[c], Dm[4 * r + c]);
            s2 = fmaf(Dm[4 * r + c], kc[c], s2);
          }
          w[r] = s2;
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
          if (lane == r) dv[((size_t)t * hv + h) * D + i0 + r0 + r] = de;
        }
        dap = warp_sum(dap);
        float* rw = red + (par * BW_WARPS + warp) * BW_RED_LD;
        *reinterpret_cast<float4*>(rw + c0) = make_float4(dqp[0], dqp[1], dqp[2], dqp[3]);
        *reinterpret_cast<float4*>(rw + D + c0) = make_float4(dkp[0], dkp[1], dkp[2], dkp[3]);
        if (lane == 0) {
          rw[2 * D] = dbp;
          rw[2 * D + 1] = dap;
        }
        __syncthreads();
        for (int x = tid; x < BW_RED; x += BW_THREADS) {  // the slice's sums over its warps, in warp order
          float s2 = 0.0f;
#pragma unroll
          for (int ww = 0; ww < BW_WARPS; ++ww) s2 += red[(par * BW_WARPS + ww) * BW_RED_LD + x];
          part[(((size_t)sl * T + t) * hv + h) * BW_RED + x] = s2;
        }
        par ^= 1;  // the next token writes the other buffer; this one is read before the next barrier
      }
    }
  }
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) dS_init[sbase + elem(r, c)] = Dm[4 * r + c];
}

// dq, dk of QK head j = the sum over its value heads and their row slices; dbeta, dg of value
// head h = the sum over its slices (dg times alpha_t).  Fixed order: value head, then slice.
__global__ void __launch_bounds__(128) k_bwd_sum(Dims d, const float* __restrict__ part, const float* __restrict__ g,
                                                 float* __restrict__ dq, float* __restrict__ dk,
                                                 float* __restrict__ dbeta, float* __restrict__ dg) {
  const int t = blockIdx.x, j = blockIdx.y, c = threadIdx.x;
  const int hq = d.h_qk, hv = d.h_v, G = hv / hq;
  const size_t T = (size_t)d.total_tokens;
  auto P = [&](int sl, int h) { return part + (((size_t)sl * T + t) * hv + h) * BW_RED; };
  float sq = 0.0f, sk = 0.0f;
  for (int gg = 0; gg < G; ++gg)
    for (int sl = 0; sl < BW_SL; ++sl) {
      const float* p = P(sl, j * G + gg);
      sq += p[c];
      sk += p[D + c];
    }
  dq[((size_t)t * hq + j) * D + c] = sq;
  dk[((size_t)t * hq + j) * D + c] = sk;
  if (c < G) {
    const int h = j * G + c;
    float sb = 0.0f, sa = 0.0f;
    for (int sl = 0; sl < BW_SL; ++sl) {
      sb += P(sl, h)[2 * D];
      sa += P(sl, h)[2 * D + 1];
    }
    dbeta[(size_t)t * hv + h] = sb;
    dg[(size_t)t * hv + h] = __expf(g[(size_t)t * hv + h]) * sa;
  }
}

}  // namespace gdn
