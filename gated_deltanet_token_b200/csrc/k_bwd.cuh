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
// rows), and warp w owns slice rows 4w .. 4w + 3, 16 elements of S or D per thread: in the
// recompute and the reverse, lane l holds columns 4l .. 4l + 3 of all four rows (the column
// sums of dq and dk stay in the thread); in the two chunk-level forward passes, lane l holds
// row l / 8 in the column groups (l % 8) + 8 m (a row product reduces over eight lanes).  Row
// dot products are warp reductions: one group per
// forward token (S_{t-1} k_t) and one per reverse token (D' k_t and <D', S_{t-1}> together, with
// D' = D + dy q^T, since <dS', S_{t-1}> = <D', S_{t-1}> - sum_r de_r (S_{t-1} k_t)_r).  The
// column sums of dq, dk and the scalars dbeta, dg are reduced over the 8 warps through shared
// memory and written per slice, one token later (three buffers, one barrier per token), so the
// sum is off the token chain; k_bwd_sum adds the slices and the value heads that share a QK
// head, in a fixed order.
//   1. Forward over the sequence, storing the state at every 64-token chunk start (global);
//      the next chunk's inputs are copied to shared memory (cp.async) during the current one.
//   2. For each chunk from the last: its k, v, g, beta go to shared memory; a forward pass over
//      the chunk keeps the state at every 8th token in shared memory; then, per 8-token
//      sub-chunk from the last, the 8 states before its tokens are recomputed into registers
//      (with S_{t-1} k_t to shared memory) and the sub-chunk's tokens are walked in reverse,
//      while the next sub-chunk's q and dy rows are copied in.  No state sequence goes
//      through global memory.
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
constexpr int BW_NRED = 3;                             // partial buffers: a token's are summed one token later
constexpr size_t BW_CK_FLOATS = (size_t)D * D;         // one checkpoint of a value head's state

// A chunk's input block (floats): k [64][128], v of the slice [64][32], g [64], beta [64].
constexpr int BWI_K = 0, BWI_V = CH * D, BWI_G = BWI_V + CH * BW_NR, BWI_B = BWI_G + CH, BWI_FLOATS = BWI_B + CH;
// Shared memory (floats): the input block; the sub-chunk checkpoints ([8][4 quads][256 threads]
// float4, a warp's accesses consecutive), which hold the second input block during the forward
// sweep; q and dy rows of a sub-chunk, double-buffered ([2][8][128], [2][8][32]); S_{t-1} k_t of
// the sub-chunk ([8 tokens][8 warps][4 rows]); the per-warp partials [3][8][BW_RED_LD].
constexpr int BWS_IN = 0, BWS_SUBCK = BWS_IN + BWI_FLOATS;
constexpr int BWS_Q = BWS_SUBCK + BW_NSUB * BW_EL * BW_THREADS, BWS_DY = BWS_Q + 2 * BW_SUB * D;
constexpr int BWS_SK = BWS_DY + 2 * BW_SUB * BW_NR, BWS_RED = BWS_SK + BW_SUB * BW_WARPS * BW_ROWS;
constexpr size_t BW_SMEM = (size_t)(BWS_RED + BW_NRED * BW_WARPS * BW_RED_LD) * 4;
static_assert(BW_SMEM <= 227 * 1024, "k_bwd shared memory");
static_assert(BWI_FLOATS <= BW_NSUB * BW_EL * BW_THREADS, "the second input block fits the sub-checkpoints");
static_assert(BWS_SUBCK % 4 == 0 && BWS_Q % 4 == 0 && BWS_DY % 4 == 0 && BWS_SK % 4 == 0 && BWS_RED % 4 == 0,
              "16-byte aligned regions");

__device__ __forceinline__ void bw_cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void bw_cp4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void bw_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bw_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// A thread's state elements as paired floats: row r, columns (0, 1) at [2 r] and (2, 3) at
// [2 r + 1], so that the row updates run as paired fp32 FMAs.
constexpr int BW_EL2 = BW_EL / 2;
__device__ __forceinline__ float2 bw_f2(float x) { return make_float2(x, x); }

// One forward token on the thread's elements: sk_r = (S k)_r, e_r = beta (v_r - alpha sk_r),
// S <- alpha S + e k^T.  k4: the thread's 4 key components; vrow: the warp's BW_ROWS values.
// Every pass runs this same arithmetic.
__device__ __forceinline__ void bw_forward_token(float2 (&S)[BW_EL2], float (&sk)[BW_ROWS], float a, float bt,
                                                 const float4 k4, const float* vrow, bool update) {
  const float2 k01 = make_float2(k4.x, k4.y), k23 = make_float2(k4.z, k4.w);
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r) {
    const float2 p = __ffma2_rn(S[2 * r + 1], k23, __fmul2_rn(S[2 * r], k01));
    sk[r] = p.x + p.y;
  }
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r) sk[r] = warp_sum(sk[r]);
  if (!update) return;
  const float2 a2 = bw_f2(a);
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r) {
    const float2 e2 = bw_f2(bt * (vrow[r] - a * sk[r]));
    S[2 * r] = __ffma2_rn(e2, k01, __fmul2_rn(a2, S[2 * r]));
    S[2 * r + 1] = __ffma2_rn(e2, k23, __fmul2_rn(a2, S[2 * r + 1]));
  }
}

// The same token in the row layout of the two chunk-level forward passes: the thread holds one
// row of the warp's four, in the 4-column groups cg + 8 m (m = 0..3, S[2 m], S[2 m + 1]), so
// that a row product reduces over eight lanes (three shuffle levels).  krow: k_t (128 floats);
// vr: v_t of the thread's row.
__device__ __forceinline__ void bw_forward_row(float2 (&S)[BW_EL2], float a, float bt, const float* krow, float vr,
                                               int cg) {
  float2 k2[BW_EL2];
#pragma unroll
  for (int m = 0; m < BW_EL2 / 2; ++m) {
    const float4 k4 = *reinterpret_cast<const float4*>(krow + 4 * (cg + 8 * m));
    k2[2 * m] = make_float2(k4.x, k4.y);
    k2[2 * m + 1] = make_float2(k4.z, k4.w);
  }
  float2 p0 = __fmul2_rn(S[0], k2[0]), p1 = __fmul2_rn(S[1], k2[1]);
#pragma unroll
  for (int x = 2; x < BW_EL2; x += 2) {
    p0 = __ffma2_rn(S[x], k2[x], p0);
    p1 = __ffma2_rn(S[x + 1], k2[x + 1], p1);
  }
  float sk = (p0.x + p0.y) + (p1.x + p1.y);
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) sk += __shfl_xor_sync(0xffffffffu, sk, o);
  const float2 e2 = bw_f2(bt * (vr - a * sk)), a2 = bw_f2(a);
#pragma unroll
  for (int x = 0; x < BW_EL2; ++x) S[x] = __ffma2_rn(e2, k2[x], __fmul2_rn(a2, S[x]));
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
  const int rr = lane >> 3, cg = lane & 7;         // row layout: slice row r0 + rr, column groups cg + 8 m
  const size_t sbase = ((size_t)n * hv + h) * D * D;
  const size_t T = (size_t)d.total_tokens;
  auto elem = [&](int r, int c) { return (size_t)(i0 + r0 + r) * D + c0 + c; };
  float* const in0 = bsm + BWS_IN;
  float* const in1 = bsm + BWS_SUBCK;  // the forward sweep's second input block
  float4* const sSub = reinterpret_cast<float4*>(bsm + BWS_SUBCK);
  float* const sQ = bsm + BWS_Q;
  float* const sDY = bsm + BWS_DY;
  float* const sSK = bsm + BWS_SK;
  float* const red = bsm + BWS_RED;
  // checkpoint of chunk ci: slot (gc0 + ci, h), slice sl, [4 quads][256 threads] float4
  auto ckp = [&](int ci) {
    return reinterpret_cast<float4*>(ck_ws + ((size_t)(gc0 + ci) * hv + h) * BW_CK_FLOATS +
                                     (size_t)sl * BW_EL * BW_THREADS) + tid;
  };
  // row r of the thread's elements is float4 number r of its slots
  auto put = [&](float4* p, const float2 (&x)[BW_EL2]) {
#pragma unroll
    for (int r = 0; r < BW_ROWS; ++r)
      p[r * BW_THREADS] = make_float4(x[2 * r].x, x[2 * r].y, x[2 * r + 1].x, x[2 * r + 1].y);
  };
  auto get = [&](const float4* p, float2 (&x)[BW_EL2]) {
#pragma unroll
    for (int r = 0; r < BW_ROWS; ++r) {
      const float4 f = p[r * BW_THREADS];
      x[2 * r] = make_float2(f.x, f.y);
      x[2 * r + 1] = make_float2(f.z, f.w);
    }
  };
  // the thread's elements of a [N][h_v][d_v][d_k] state (or zeros for a null pointer)
  auto load_state = [&](const float* src, float2 (&x)[BW_EL2]) {
#pragma unroll
    for (int r = 0; r < BW_ROWS; ++r) {
      const float4 f = src ? *reinterpret_cast<const float4*>(src + sbase + elem(r, 0)) : make_float4(0, 0, 0, 0);
      x[2 * r] = make_float2(f.x, f.y);
      x[2 * r + 1] = make_float2(f.z, f.w);
    }
  };
  // row layout: the thread's elements of a [N][h_v][d_v][d_k] state (or zeros for a null pointer)
  auto load_state_row = [&](const float* src, float2 (&x)[BW_EL2]) {
#pragma unroll
    for (int m = 0; m < BW_EL2 / 2; ++m) {
      const float4 f = src ? *reinterpret_cast<const float4*>(src + sbase + (size_t)(i0 + r0 + rr) * D + 4 * (cg + 8 * m))
                           : make_float4(0, 0, 0, 0);
      x[2 * m] = make_float2(f.x, f.y);
      x[2 * m + 1] = make_float2(f.z, f.w);
    }
  };
  // sub-checkpoint sc in shared memory: [32 rows][32 four-column groups] float4, written in the
  // row layout and read in the column layout, both as 128 contiguous bytes per eight lanes
  auto sub_unit = [&](int sc, int row, int grp) { return sSub + ((sc * BW_NR + row) * (D / 4) + grp); };
  // copies (cp.async, not committed) of the L tokens from t0 into an input block
  auto load_inputs = [&](float* blk, int t0, int L) {
    for (int i = tid; i < L * (D / 4); i += BW_THREADS)
      bw_cp16(blk + BWI_K + 4 * i, kh + ((size_t)(t0 + i / (D / 4)) * hq + j) * D + 4 * (i % (D / 4)));
    for (int i = tid; i < L * (BW_NR / 4); i += BW_THREADS)
      bw_cp16(blk + BWI_V + 4 * i, v + ((size_t)(t0 + i / (BW_NR / 4)) * hv + h) * D + i0 + 4 * (i % (BW_NR / 4)));
    for (int i = tid; i < L; i += BW_THREADS) {
      bw_cp4(blk + BWI_G + i, g + (size_t)(t0 + i) * hv + h);
      bw_cp4(blk + BWI_B + i, beta + (size_t)(t0 + i) * hv + h);
    }
  };
  // copies of the q and dy rows of nt tokens from t0 into buffer b
  auto load_qdy = [&](int b, int t0, int nt) {
    for (int i = tid; i < nt * (D / 4); i += BW_THREADS)
      bw_cp16(sQ + b * BW_SUB * D + 4 * i, qh + ((size_t)(t0 + i / (D / 4)) * hq + j) * D + 4 * (i % (D / 4)));
    for (int i = tid; i < nt * (BW_NR / 4); i += BW_THREADS)
      bw_cp16(sDY + b * BW_SUB * BW_NR + 4 * i,
              dy + ((size_t)(t0 + i / (BW_NR / 4)) * hv + h) * D + i0 + 4 * (i % (BW_NR / 4)));
  };
  auto fwd_row = [&](float2 (&S)[BW_EL2], const float* blk, int tt) {
    bw_forward_row(S, __expf(blk[BWI_G + tt]), blk[BWI_B + tt], blk + BWI_K + tt * D, blk[BWI_V + tt * BW_NR + r0 + rr],
                   cg);
  };

  // ---- 1. forward, a checkpoint at every chunk start (row layout) -------------------------
  float2 S[BW_EL2];
  load_state_row(init_state, S);
  if (nchunks > 0) load_inputs(in0, ts, min(CH, te - ts));
  bw_commit();
  for (int ci = 0; ci < nchunks; ++ci) {
    const int t0 = ts + ci * CH, L = min(CH, te - t0);
    float* blk = (ci & 1) ? in1 : in0;
    put(ckp(ci), S);
    if (ci + 1 < nchunks) load_inputs((ci & 1) ? in0 : in1, t0 + CH, min(CH, te - t0 - CH));
    bw_commit();
    bw_wait<1>();  // this chunk's copies landed (the next chunk's may be in flight)
    __syncthreads();
    for (int tt = 0; tt < L; ++tt) fwd_row(S, blk, tt);
    __syncthreads();  // the next iteration copies into this block
  }

  // ---- 2. reverse, chunk by chunk from the last ---------------------------------------------
  float2 Dm[BW_EL2];
  load_state(dS_final, Dm);
  // the slice's partials of token tp in buffer rb: summed over the warps, in warp order
  auto reduce = [&](int rb, int tp) {
    for (int x = tid; x < BW_RED; x += BW_THREADS) {
      float s2 = 0.0f;
#pragma unroll
      for (int ww = 0; ww < BW_WARPS; ++ww) s2 += red[(rb * BW_WARPS + ww) * BW_RED_LD + x];
      part[(((size_t)sl * T + tp) * hv + h) * BW_RED + x] = s2;
    }
  };
  int kred = 0;      // reverse tokens done: the partial buffer of the next is kred % 3
  int pend = -1;     // the token whose partials wait in buffer (kred + 2) % 3
  int nsub = 0;      // sub-chunks done: the q / dy buffer of the next is nsub & 1
  if (nchunks > 0) {
    const int t0 = ts + (nchunks - 1) * CH, L = te - t0, tb = (L - 1) / BW_SUB * BW_SUB;
    load_qdy(0, t0 + tb, L - tb);
  }
  bw_commit();
  for (int ci = nchunks - 1; ci >= 0; --ci) {
    const int t0 = ts + ci * CH, L = min(CH, te - t0);
    __syncthreads();  // the later chunk's inputs and sub-checkpoints are no longer read
    load_inputs(in0, t0, L);
    bw_commit();
    get(ckp(ci), S);
    bw_wait<0>();
    __syncthreads();
    // the state before every 8th token, to the sub-checkpoints (row layout)
    for (int tt = 0; tt < L; ++tt) {
      if (tt % BW_SUB == 0) {
#pragma unroll
        for (int m = 0; m < BW_EL2 / 2; ++m)
          *sub_unit(tt / BW_SUB, r0 + rr, cg + 8 * m) = make_float4(S[2 * m].x, S[2 * m].y, S[2 * m + 1].x, S[2 * m + 1].y);
      }
      fwd_row(S, in0, tt);
    }
    __syncthreads();  // the sub-checkpoints are read by other threads (column layout)
    for (int sc = (L + BW_SUB - 1) / BW_SUB - 1; sc >= 0; --sc) {
      const int tb = sc * BW_SUB, nt = min(BW_SUB, L - tb);  // block-uniform
      const int b = nsub & 1;
      // the next sub-chunk's q and dy rows into the other buffer (read by the previous one,
      // whose last token's barrier every thread has passed)
      const bool more = sc > 0 || ci > 0;
      if (sc > 0) load_qdy(b ^ 1, t0 + tb - BW_SUB, BW_SUB);
      else if (ci > 0) load_qdy(b ^ 1, t0 - BW_SUB, BW_SUB);
      bw_commit();
      // St[i]: the state before token tb + i; S_{t-1} k_t of every token to shared memory
      float2 St[BW_SUB][BW_EL2];
#pragma unroll
      for (int r = 0; r < BW_ROWS; ++r) {
        const float4 f = *sub_unit(sc, r0 + r, lane);
        St[0][2 * r] = make_float2(f.x, f.y);
        St[0][2 * r + 1] = make_float2(f.z, f.w);
      }
#pragma unroll
      for (int i = 0; i < BW_SUB; ++i) {
        if (i < nt) {
          const int tt = tb + i;
          float sk[BW_ROWS];
          if (i + 1 < BW_SUB) {
#pragma unroll
            for (int x = 0; x < BW_EL2; ++x) St[i + 1][x] = St[i][x];
            bw_forward_token(St[i + 1], sk, __expf(in0[BWI_G + tt]), in0[BWI_B + tt],
                             *reinterpret_cast<const float4*>(in0 + BWI_K + tt * D + c0),
                             in0 + BWI_V + tt * BW_NR + r0, i + 1 < nt);
          } else {
            float2 Sx[BW_EL2];
#pragma unroll
            for (int x = 0; x < BW_EL2; ++x) Sx[x] = St[i][x];
            bw_forward_token(Sx, sk, 0.0f, 0.0f, *reinterpret_cast<const float4*>(in0 + BWI_K + tt * D + c0),
                             in0 + BWI_V + tt * BW_NR + r0, false);
          }
          if (lane == 0)
            *reinterpret_cast<float4*>(sSK + (i * BW_WARPS + warp) * BW_ROWS) = make_float4(sk[0], sk[1], sk[2], sk[3]);
        }
      }
      if (more) bw_wait<1>();  // this sub-chunk's q / dy copies landed
      else bw_wait<0>();
      __syncthreads();
      const float* qb = sQ + b * BW_SUB * D;
      const float* yb = sDY + b * BW_SUB * BW_NR;
#pragma unroll
      for (int i = BW_SUB - 1; i >= 0; --i) {
        if (i >= nt) continue;
        const int tt = tb + i, t = t0 + tt;
        const float2* Sprev = St[i];
        const float a = __expf(in0[BWI_G + tt]), bt = in0[BWI_B + tt];
        const float4 k4 = *reinterpret_cast<const float4*>(in0 + BWI_K + tt * D + c0);
        const float4 q4 = *reinterpret_cast<const float4*>(qb + i * D + c0);
        const float4 s4 = *reinterpret_cast<const float4*>(sSK + (i * BW_WARPS + warp) * BW_ROWS);
        const float* vrow = in0 + BWI_V + tt * BW_NR + r0;
        const float* yrow = yb + i * BW_NR + r0;
        const float2 k01 = make_float2(k4.x, k4.y), k23 = make_float2(k4.z, k4.w);
        const float2 q01 = make_float2(q4.x, q4.y), q23 = make_float2(q4.z, q4.w), a2 = bw_f2(a);
        const float sk[BW_ROWS] = {s4.x, s4.y, s4.z, s4.w};
        // e_t = v_t - alpha (S_{t-1} k_t);  dq partial = S_t^T dy (S_t = alpha S_{t-1} + beta e k^T)
        // D' = D + dy q^T;  w = D' k;  P = <D', S_{t-1}>  (one reduction group)
        float e[BW_ROWS], w[BW_ROWS + 1];
        float2 dq01 = make_float2(0.0f, 0.0f), dq23 = dq01, pp = dq01;
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) {
          e[r] = vrow[r] - a * sk[r];
          const float2 gy2 = bw_f2(yrow[r]), be2 = bw_f2(bt * e[r]);
          dq01 = __ffma2_rn(gy2, __ffma2_rn(a2, Sprev[2 * r], __fmul2_rn(be2, k01)), dq01);
          dq23 = __ffma2_rn(gy2, __ffma2_rn(a2, Sprev[2 * r + 1], __fmul2_rn(be2, k23)), dq23);
          Dm[2 * r] = __ffma2_rn(gy2, q01, Dm[2 * r]);
          Dm[2 * r + 1] = __ffma2_rn(gy2, q23, Dm[2 * r + 1]);
          const float2 wv = __ffma2_rn(Dm[2 * r + 1], k23, __fmul2_rn(Dm[2 * r], k01));
          w[r] = wv.x + wv.y;
          pp = __ffma2_rn(Dm[2 * r], Sprev[2 * r], pp);
          pp = __ffma2_rn(Dm[2 * r + 1], Sprev[2 * r + 1], pp);
        }
        w[BW_ROWS] = pp.x + pp.y;
#pragma unroll
        for (int r = 0; r <= BW_ROWS; ++r) w[r] = warp_sum(w[r]);
        // de = beta w (= dv);  dbeta = e . w;  dk partial = beta D'^T e - alpha S_{t-1}^T de;
        // dS' = D' - de k^T;  dalpha = <dS', S_{t-1}> = P - de . (S_{t-1} k);  D <- alpha dS'
        float2 dk01 = make_float2(0.0f, 0.0f), dk23 = dk01;
        float dbp = 0.0f, dap = w[BW_ROWS];
#pragma unroll
        for (int r = 0; r < BW_ROWS; ++r) {
          const float de = bt * w[r];
          dbp = fmaf(e[r], w[r], dbp);
          dap = fmaf(-de, sk[r], dap);
          const float2 be2 = bw_f2(bt * e[r]), mdea = bw_f2(-de * a), mde = bw_f2(-de);
          dk01 = __ffma2_rn(be2, Dm[2 * r], __ffma2_rn(mdea, Sprev[2 * r], dk01));
          dk23 = __ffma2_rn(be2, Dm[2 * r + 1], __ffma2_rn(mdea, Sprev[2 * r + 1], dk23));
          Dm[2 * r] = __fmul2_rn(a2, __ffma2_rn(mde, k01, Dm[2 * r]));
          Dm[2 * r + 1] = __fmul2_rn(a2, __ffma2_rn(mde, k23, Dm[2 * r + 1]));
          if (lane == r) dv[((size_t)t * hv + h) * D + i0 + r0 + r] = de;
        }
        const float dqp[4] = {dq01.x, dq01.y, dq23.x, dq23.y}, dkp[4] = {dk01.x, dk01.y, dk23.x, dk23.y};
        float* rw = red + ((kred % BW_NRED) * BW_WARPS + warp) * BW_RED_LD;
        *reinterpret_cast<float4*>(rw + c0) = make_float4(dqp[0], dqp[1], dqp[2], dqp[3]);
        *reinterpret_cast<float4*>(rw + D + c0) = make_float4(dkp[0], dkp[1], dkp[2], dkp[3]);
        if (lane == 0) {
          rw[2 * D] = dbp;
          rw[2 * D + 1] = dap;
        }
        __syncthreads();
        if (pend >= 0) reduce((kred + BW_NRED - 1) % BW_NRED, pend);
        pend = t;
        ++kred;
      }
      ++nsub;
    }
  }
  __syncthreads();
  if (pend >= 0) reduce((kred + BW_NRED - 1) % BW_NRED, pend);
#pragma unroll
  for (int r = 0; r < BW_ROWS; ++r)
    *reinterpret_cast<float4*>(dS_init + sbase + elem(r, 0)) =
        make_float4(Dm[2 * r].x, Dm[2 * r].y, Dm[2 * r + 1].x, Dm[2 * r + 1].y);
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
