// k_chunk_tc.cuh -- chunked gated delta rule on tcgen05 tensor cores (bf16-input path).
//
// Same chunk algebra as k_chunk_simt.cuh (an exact rewrite of the six steps of the
// "Qwen3-Next 80B-A3B" field guide, §02; the state carry is the chunk-loop update of the
// "Qwen3.8-Flash-Next" model notes in column-vector form), regrouped so that every
// contraction is an M = 128 tcgen05 MMA:
//
//   R   = diag(beta) (V - diag(e^gamma) K S^T)              [U = T R, T = (I + A)^-1]
//   [U ; M o QK^T U] = [T ; P] R,   P = (M o QK^T) T        (one MMA, 128 x nv x 64)
//   Y   = diag(e^gamma) Q S^T + (M o QK^T) U
//   S^T <- e^{gamma_L} S^T + K^T diag(e^{gamma_L - gamma}) U
//   [K S^T ; Q S^T] = [K ; Q] S^T                            (one MMA, 128 x nv x 128)
//
// Every tensor-core product is taken in three bf16 terms, a_hi b_hi + a_hi b_lo + a_lo b_hi,
// with x = hi + lo the bf16 split of an fp32 value: plain bf16 operands lose ~2^-9 per
// element, which the scale-invariant output norm amplifies on tokens with a small y_raw;
// the split keeps the products at ~2^-17 relative error.
//
// Phase A (k_chunkprep_tc, parallel over chunks x QK heads): conv + SiLU + L2 norm of q, k;
// the [K;Q] hi/lo tile (stored to the workspace with one bulk copy); [K;Q] K^T on tcgen05;
// per value head: gates, gamma, A, M o QK^T, T = (I + A)^-1 (blocked 16 x 16 forward
// substitution), P = (M o QK^T) T, and the [T;P] hi/lo tile.
// Phase B (k_chunkscan_tc, sequential over one sequence's chunks, parallel over value
// heads and 32-row slices of the state): the three MMA rounds above per chunk, with the
// next chunk's tiles bulk-copied into a second stage while the current one computes.
#pragma once
#include "gdn_common.cuh"
#include "tc_ptx.cuh"

namespace gdn {

constexpr int TC_NV = 32;                            // state rows (value components) per phase-B CTA
constexpr uint32_t KQ_TILE = 128 * 128 * 2;          // one bf16 tile of [K;Q] (hi or lo): 32 KB
constexpr uint32_t KQ_BYTES = 2 * KQ_TILE;           // per (chunk, QK head)
constexpr uint32_t TP_TILE = 128 * 64 * 2;           // one bf16 tile of [T;P]: 16 KB
constexpr uint32_t TP_BYTES = 2 * TP_TILE;           // per (chunk, value head)
constexpr uint32_t GB_FLOATS = 128;                  // gamma[64], beta[64] per (chunk, value head)
constexpr uint32_t LBO128 = 2048;                    // K-direction core stride of 128-row tiles

// Byte offset of element (r, k) in a K-major no-swizzle tile with 128 rows.
__device__ __forceinline__ uint32_t kmaj128(int r, int k) {
  return (uint32_t)((k >> 3) * LBO128 + (r >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2);
}
// Byte offset of the 16-byte chunk (k row, n-block nb) of an MN-major tile with K rows
// (LBO = 128: K groups adjacent; SBO = K / 8 * 128).
__device__ __forceinline__ uint32_t mnmaj(int k, int nb, int K) {
  return (uint32_t)(nb * (K / 8) * 128 + (k >> 3) * 128 + (k & 7) * 16);
}

// ======================================================================================
// Self-test of the four operand-layout combinations the kernels use (diagnostic entry
// point gdn_selftest_tc).  case 0: A K-major 128x128, B = first 64 rows of A (K-major);
// case 1: A K-major 128x128, B MN-major K=128 N=32; case 2: A K-major 128x64, B MN-major
// K=64 N=32; case 3: A = transpose of rows 0..63 of a K-major 128-row tile (MN-major
// view), B MN-major K=64 N=32.  out[0] = max |D - ref|, out[1] = max |ref|.
// ======================================================================================
__device__ __forceinline__ float st_val(uint32_t i, uint32_t salt) {
  uint32_t x = i * 2654435761u ^ (salt * 0x9E3779B9u + 0x85EBCA6Bu);
  x ^= x >> 15; x *= 0x2C1B3C6Du; x ^= x >> 12; x *= 0x297A2D39u; x ^= x >> 15;
  const float u = (float)(x & 0xFFFFFF) * (1.0f / 16777216.0f) * 2.0f - 1.0f;
  return ldexpf(u, -(int)((x >> 24) & 7));
}

template <int CASE>
__global__ void __launch_bounds__(128) k_selftest_umma(float* out) {
  constexpr int N = CASE == 0 ? 64 : 32;
  constexpr int K = (CASE == 0 || CASE == 1) ? 128 : 64;
  constexpr int ROWS_A = 128;  // rows of the physical A tile (case 3: the 128-row tile)
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* Ahi = sm;
  uint8_t* Alo = sm + 32768;
  uint8_t* Bhi = sm + 65536;
  uint8_t* Blo = sm + 65536 + 16384;
  __shared__ uint64_t mbar;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a_cols = CASE == 3 ? 128 : K;  // K-major physical columns of the A tile
  // logical A[m][k] and B[k][n]
  auto Aval = [&](int m, int k) { return CASE == 3 ? st_val(k * 128 + m, 11u) : st_val(m * 1024 + k, 1u + CASE); };
  auto Bval = [&](int k, int n) { return CASE == 0 ? Aval(n, k) : st_val(k * 64 + n, 7u + CASE); };
  // physical A tile (K-major, 128 rows): case 3 stores X[s][j] = A[j][s] at (r = s, k = j)
  for (int idx = tid; idx < ROWS_A * a_cols; idx += 128) {
    const int r = idx / a_cols, c = idx % a_cols;
    float v = CASE == 3 ? (r < 64 ? Aval(c, r) : 0.0f) : Aval(r, c);
    uint16_t h, l;
    tc::split2(v, h, l);
    *reinterpret_cast<uint16_t*>(Ahi + kmaj128(r, c)) = h;
    *reinterpret_cast<uint16_t*>(Alo + kmaj128(r, c)) = l;
  }
  if (CASE != 0) {  // MN-major B tile [K][N]
    for (int idx = tid; idx < K * N; idx += 128) {
      const int kk = idx / N, n = idx % N;
      uint16_t h, l;
      tc::split2(Bval(kk, n), h, l);
      const uint32_t off = mnmaj(kk, n >> 3, K) + (n & 7) * 2;
      *reinterpret_cast<uint16_t*>(Bhi + off) = h;
      *reinterpret_cast<uint16_t*>(Blo + off) = l;
    }
  }
  if (tid == 0) {
    tc::mbar_init(tc::smem_u32(&mbar), 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(&tslot), 64);
    tc::tmem_relinquish();
  }
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = tslot;
  if (tid == 0) {
    constexpr uint32_t idesc = tc::idesc_bf16(128, N, CASE == 3 ? 1 : 0, CASE == 0 ? 0 : 1);
    const uint32_t a0[2] = {tc::smem_u32(Ahi), tc::smem_u32(Alo)};
    const uint32_t b0[2] = {CASE == 0 ? tc::smem_u32(Ahi) : tc::smem_u32(Bhi),
                            CASE == 0 ? tc::smem_u32(Alo) : tc::smem_u32(Blo)};
    // A: K-major (LBO 2048, SBO 128) or, case 3, MN-major view (SBO 2048, LBO 128).
    const uint32_t a_lbo = CASE == 3 ? 128 : LBO128, a_sbo = CASE == 3 ? LBO128 : 128;
    const uint32_t b_lbo = CASE == 0 ? LBO128 : 128, b_sbo = CASE == 0 ? 128 : (K / 8) * 128;
    for (int ks = 0; ks < K / 16; ++ks) {
      for (int term = 0; term < 3; ++term) {
        const int ai = term == 2 ? 1 : 0, bi = term == 1 ? 1 : 0;
        const uint64_t ad = tc::sdesc(a0[ai] + ks * 2 * a_lbo, a_lbo, a_sbo);
        const uint64_t bd = tc::sdesc(b0[bi] + ks * 2 * b_lbo, b_lbo, b_sbo);
        tc::umma_bf16(tbase, ad, bd, idesc, (ks | term) != 0);
      }
    }
    tc::umma_commit(tc::smem_u32(&mbar));
  }
  const bool ok = tc::mbar_wait(tc::smem_u32(&mbar), 0);
  tc::tc_fence_after();
  const int m = warp * 32 + lane;
  float err = 0.0f, mag = 0.0f;
  if (ok) {
    for (int n0 = 0; n0 < N; n0 += 32) {
      uint32_t r[32];
      tc::tmem_ld32(tbase + ((uint32_t)(warp * 32) << 16) + n0, r);
      tc::tmem_wait_ld();
      for (int c = 0; c < 32; ++c) {
        const int n = n0 + c;
        float ref = 0.0f;
        for (int kk = 0; kk < K; ++kk) {
          uint16_t ah, al, bh, bl;
          tc::split2(Aval(m, kk), ah, al);
          tc::split2(Bval(kk, n), bh, bl);
          const float fah = bf2f(ah), fal = bf2f(al), fbh = bf2f(bh), fbl = bf2f(bl);
          ref = fmaf(fah, fbh, fmaf(fah, fbl, fmaf(fal, fbh, ref)));
        }
        err = fmaxf(err, fabsf(__uint_as_float(r[c]) - ref));
        mag = fmaxf(mag, fabsf(ref));
      }
    }
  } else {
    err = __int_as_float(0x7f800000);
    atomicExch(&g_gdn_status, -7);
  }
  atomicMax(reinterpret_cast<int*>(out), __float_as_int(err));
  atomicMax(reinterpret_cast<int*>(out + 1), __float_as_int(mag));
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 64);
}

// ======================================================================================
// Phase A
// ======================================================================================
constexpr size_t PA_TC_SMEM = 65536 + 64 * 64 * 4 + TP_BYTES + 2 * 64 * 4;

// Shared-memory fp32 64 x 64 matrices in phase A use pitch 64 with the column index
// XOR-swizzled by the row's 4-bit group, so row-wise and column-wise sweeps hit
// different banks.
__device__ __forceinline__ int sw64(int t, int s) { return t * 64 + (s ^ ((t & 7) << 2)); }

__global__ void __launch_bounds__(256, 2)
    k_chunkprep_tc(Dims d, const ChunkEntry* __restrict__ tab, const uint16_t* __restrict__ q,
                   const uint16_t* __restrict__ k, const float* __restrict__ a,
                   const float* __restrict__ b, const float* __restrict__ A_log,
                   const float* __restrict__ dt_bias, const float* __restrict__ conv_w,
                   uint8_t* __restrict__ kq_ws, uint8_t* __restrict__ tp_ws, float* __restrict__ gb_ws) {
  const ChunkEntry e = tab[blockIdx.x];
  if (e.len == 0) return;
  const int j = blockIdx.y, hq = d.h_qk, hv = d.h_v, G = hv / hq, L = e.len;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* kq_hi = sm;                        // [K;Q] tile, hi
  uint8_t* kq_lo = sm + KQ_TILE;              // [K;Q] tile, lo
  float* KK = reinterpret_cast<float*>(sm);   // aliases the tile once it is consumed
  float* QK = KK + 64 * 64;
  float* Am = QK + 64 * 64;
  float* Mq = Am + 64 * 64;
  float* Tm = reinterpret_cast<float*>(sm + 65536);
  uint8_t* tp = sm + 65536 + 64 * 64 * 4;     // [T;P] staging: hi then lo
  float* gs = reinterpret_cast<float*>(tp + TP_BYTES);
  float* bs = gs + 64;
  __shared__ uint64_t mbar;
  __shared__ uint32_t tslot;
  __shared__ int s_abort;

  if (tid == 0) {
    s_abort = 0;
    tc::mbar_init(tc::smem_u32(&mbar), 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(&tslot), 64);
    tc::tmem_relinquish();
  }

  // ---- conv + SiLU + L2 norm of the chunk's q and k rows into the [K;Q] tile -------------
  // warp w: tokens 8w .. 8w+7, lane: channels 4 lane .. 4 lane + 3; rows 0..63 are K, 64..127 Q.
  {
    const int tb = warp * 8, c0 = lane * 4;
#pragma unroll
    for (int st = 0; st < 2; ++st) {  // st 0: k (rows 0..63), st 1: q (rows 64..127)
      const uint16_t* src = st ? q : k;
      const size_t ch0 = st ? (size_t)j * D : (size_t)(hq + j) * D;
      float w[4][4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 t4 = *reinterpret_cast<const float4*>(conv_w + (ch0 + c0 + c) * 4);
        w[c][0] = t4.x; w[c][1] = t4.y; w[c][2] = t4.z; w[c][3] = t4.w;
      }
      float4 x[11];
#pragma unroll
      for (int p = 0; p < 11; ++p) {
        const int tc_ = tb - 3 + p;
        const long tg = (long)e.t0 + tc_;
        const bool ok = tc_ < L && tg >= e.seq_start;
        x[p] = ok ? load4<true>(src, ((size_t)tg * hq + j) * D + c0) : make_float4(0, 0, 0, 0);
      }
      const float scale = st ? d.q_scale : 1.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = tb + i;
        float r[4] = {0, 0, 0, 0};
        if (t < L) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float acc = fmaf(w[c][3], comp(x[i + 3], c),
                                   fmaf(w[c][2], comp(x[i + 2], c),
                                        fmaf(w[c][1], comp(x[i + 1], c), w[c][0] * comp(x[i], c))));
            r[c] = silu_f(acc);
          }
        }
        const float ss = warp_sum(r[0] * r[0] + r[1] * r[1] + r[2] * r[2] + r[3] * r[3]);
        const float inv = t < L ? scale / sqrtf(ss + d.l2_eps) : 0.0f;
        uint16_t h[4], l[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::split2(r[c] * inv, h[c], l[c]);
        const int row = st * 64 + t;
        const uint32_t off = kmaj128(row, c0);  // c0 % 8 in {0, 4}: 8-byte half of a core row
        *reinterpret_cast<uint2*>(kq_hi + off) = make_uint2(h[0] | (uint32_t(h[1]) << 16), h[2] | (uint32_t(h[3]) << 16));
        *reinterpret_cast<uint2*>(kq_lo + off) = make_uint2(l[0] | (uint32_t(l[1]) << 16), l[2] | (uint32_t(l[3]) << 16));
      }
    }
  }
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = tslot;
  uint8_t* kq_dst = kq_ws + ((size_t)blockIdx.x * hq + j) * KQ_BYTES;
  if (tid == 0) {
    tc::bulk_s2g(kq_dst, tc::smem_u32(sm), KQ_BYTES);
    tc::bulk_commit();
    // D[128 x 64] = [K;Q] (K-major, 128 x 128) x K^T (B = rows 0..63 of the tile, K-major)
    constexpr uint32_t idesc = tc::idesc_bf16(128, 64, 0, 0);
    const uint32_t base[2] = {tc::smem_u32(kq_hi), tc::smem_u32(kq_lo)};
    for (int ks = 0; ks < 8; ++ks)
      for (int term = 0; term < 3; ++term) {
        const int ai = term == 2, bi = term == 1;
        tc::umma_bf16(tbase, tc::sdesc(base[ai] + ks * 2 * LBO128, LBO128, 128),
                      tc::sdesc(base[bi] + ks * 2 * LBO128, LBO128, 128), idesc, (ks | term) != 0);
      }
    tc::umma_commit(tc::smem_u32(&mbar));
  }
  if (!tc::mbar_wait(tc::smem_u32(&mbar), 0)) {
    s_abort = 1;
    atomicExch(&g_gdn_status, -7);
  }
  tc::tc_fence_after();
  if (tid == 0) tc::bulk_wait_read_all();  // the tile may now be overwritten
  __syncthreads();
  const bool aborted = s_abort != 0;
  // TMEM rows 0..63: K K^T, rows 64..127: Q K^T (warps 0..3, one row per thread)
  uint32_t r0[32], r1[32];
  if (warp < 4) {
    const uint32_t ta = tbase + ((uint32_t)(warp * 32) << 16);
    tc::tmem_ld32(ta, r0);
    tc::tmem_ld32(ta + 32, r1);
    tc::tmem_wait_ld();
  }
  tc::tc_fence_before();
  __syncthreads();  // every read of the tile (MMA, bulk store) is over: alias it
  if (warp < 4 && !aborted) {
    const int row = tid;
    float* dst = row < 64 ? KK : QK;
    const int t = row & 63;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      dst[sw64(t, c)] = __uint_as_float(r0[c]);
      dst[sw64(t, 32 + c)] = __uint_as_float(r1[c]);
    }
  }
  __syncthreads();

  // ---- per value head: gates, A, M o QK^T, T = (I + A)^-1, P = (M o QK^T) T ---------------
  for (int g = 0; g < G && !aborted; ++g) {
    const int h = j * G + g;
    if (warp == 0) {
      float g0 = 0.0f, g1 = 0.0f, b0 = 0.0f, b1 = 0.0f;
      if (lane < L) {
        const size_t o = (size_t)(e.t0 + lane) * hv + h;
        g0 = decay_gate_f(a[o], A_log[h], dt_bias[h]);
        b0 = sigmoid_f(b[o]);
      }
      if (lane + 32 < L) {
        const size_t o = (size_t)(e.t0 + lane + 32) * hv + h;
        g1 = decay_gate_f(a[o], A_log[h], dt_bias[h]);
        b1 = sigmoid_f(b[o]);
      }
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, g0, o);
        const float y1 = __shfl_up_sync(0xffffffffu, g1, o);
        if (lane >= o) { g0 += y0; g1 += y1; }
      }
      g1 += __shfl_sync(0xffffffffu, g0, 31);
      gs[lane] = g0; gs[lane + 32] = g1;
      bs[lane] = b0; bs[lane + 32] = b1;
      float* gb = gb_ws + ((size_t)blockIdx.x * hv + h) * GB_FLOATS;
      gb[lane] = g0; gb[lane + 32] = g1;
      gb[64 + lane] = b0; gb[96 + lane] = b1;
    }
    __syncthreads();
    for (int idx = tid; idx < 64 * 64; idx += 256) {
      const int t = idx >> 6, s = idx & 63;
      const float dec = s <= t ? expf(gs[t] - gs[s]) : 0.0f;  // mask before exp
      Am[sw64(t, s)] = s < t ? bs[t] * dec * KK[sw64(t, s)] : 0.0f;
      Mq[sw64(t, s)] = dec * QK[sw64(t, s)];
    }
    __syncthreads();
    // T = (I + A)^-1, blocked by 16 x 16: diagonal blocks by forward substitution ...
    if (tid < 64) {
      const int blk = tid >> 4, c = tid & 15, o = blk * 16;
      float x[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        float v = (t == c) ? 1.0f : 0.0f;
#pragma unroll
        for (int r = 0; r < t; ++r) v = fmaf(-Am[sw64(o + t, o + r)], x[r], v);
        x[t] = v;
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) Tm[sw64(o + t, o + c)] = x[t];
    }
    for (int idx = tid; idx < 64 * 64; idx += 256) {  // zero the strict upper triangle of blocks
      const int t = idx >> 6, s = idx & 63;
      if ((s >> 4) > (t >> 4)) Tm[sw64(t, s)] = 0.0f;
    }
    __syncthreads();
    // ... then block (bi, bj), bi > bj, by distance: T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj.
    for (int dist = 1; dist < 4; ++dist) {
      const int nblk = 4 - dist;
      int ti = -1, tj = -1;
      if (tid < nblk * 64) {  // thread: (block bj, row-in-block rr, 4 columns)
        const int bj = tid >> 6, bi = bj + dist, rr = (tid >> 2) & 15, cq = (tid & 3) * 4;
        ti = bi * 16 + rr;
        tj = bj * 16 + cq;
        float w4[4] = {0, 0, 0, 0};
        // W = sum_{k=bj}^{bi-1} A_{bi,k} T_{k,bj}, row rr of block bi, columns cq..cq+3
        for (int kb = bj; kb < bi; ++kb)
#pragma unroll 4
          for (int kk = 0; kk < 16; ++kk) {
            const float av = Am[sw64(ti, kb * 16 + kk)];
#pragma unroll
            for (int c = 0; c < 4; ++c) w4[c] = fmaf(av, Tm[sw64(kb * 16 + kk, tj + c)], w4[c]);
          }
        // stage W in the strict upper triangle of Am (read by nobody), transposed
#pragma unroll
        for (int c = 0; c < 4; ++c) Am[sw64(tj + c, ti)] = w4[c];
      }
      __syncthreads();
      float res[4] = {0, 0, 0, 0};
      if (tid < nblk * 64) {
        const int bi = (tid >> 6) + dist, rr = (tid >> 2) & 15;
        // T_ij[rr][c] = -sum_m T_ii[rr][m] W[m][c]
        for (int m = 0; m <= rr; ++m) {
          const float tv = Tm[sw64(bi * 16 + rr, bi * 16 + m)];
#pragma unroll
          for (int c = 0; c < 4; ++c) res[c] = fmaf(-tv, Am[sw64(tj + c, bi * 16 + m)], res[c]);
        }
      }
      __syncthreads();
      if (tid < nblk * 64) {
#pragma unroll
        for (int c = 0; c < 4; ++c) Tm[sw64(ti, tj + c)] = res[c];
      }
      __syncthreads();
    }
    // P = (M o QK^T) T, and the [T;P] hi/lo tile: thread (t = tid / 4, 16 columns)
    {
      const int t = tid >> 2, s0 = (tid & 3) * 16;
      float p[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) p[c] = 0.0f;
      for (int r = s0; r <= t; ++r) {  // P[t][s] = sum_{s <= r <= t} Mq[t][r] T[r][s]
        const float mv = Mq[sw64(t, r)];
#pragma unroll
        for (int c = 0; c < 16; ++c) p[c] = fmaf(mv, Tm[sw64(r, s0 + c)], p[c]);
      }
      float tv[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) tv[c] = Tm[sw64(t, s0 + c)];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint4 th, tl, ph, pl;
        tc::split8(tv + half * 8, th, tl);
        tc::split8(p + half * 8, ph, pl);
        const int kcol = s0 + half * 8;
        *reinterpret_cast<uint4*>(tp + kmaj128(t, kcol)) = th;
        *reinterpret_cast<uint4*>(tp + TP_TILE + kmaj128(t, kcol)) = tl;
        *reinterpret_cast<uint4*>(tp + kmaj128(64 + t, kcol)) = ph;
        *reinterpret_cast<uint4*>(tp + TP_TILE + kmaj128(64 + t, kcol)) = pl;
      }
    }
    tc::fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
      tc::bulk_s2g(tp_ws + ((size_t)blockIdx.x * hv + h) * TP_BYTES, tc::smem_u32(tp), TP_BYTES);
      tc::bulk_commit();
      tc::bulk_wait_read_all();  // staging reusable for the next head
    }
    __syncthreads();
  }
  if (tid == 0) tc::bulk_wait_all();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 64);
}

// ======================================================================================
// Phase B
// ======================================================================================
struct PBStage {  // byte offsets inside one stage
  static constexpr uint32_t KQ = 0;
  static constexpr uint32_t TP = KQ_BYTES;
  static constexpr uint32_t GB = KQ_BYTES + TP_BYTES;
  static constexpr uint32_t BYTES = KQ_BYTES + TP_BYTES + GB_FLOATS * 4;
};
constexpr uint32_t PB_S_TILE = 128 * TC_NV * 2;  // S^T operand (K = 128, N = nv), one of hi/lo
constexpr uint32_t PB_R_TILE = 64 * TC_NV * 2;   // R / U-tilde operand (K = 64, N = nv)
constexpr size_t PB_TC_SMEM = 2 * (size_t)PBStage::BYTES + 2 * PB_S_TILE + 2 * PB_R_TILE;

__global__ void __launch_bounds__(128, 1)
    k_chunkscan_tc(Dims d, const int* __restrict__ cu, const int* __restrict__ seq_chunk0,
                   const uint16_t* __restrict__ v, const float* __restrict__ conv_w,
                   const uint8_t* __restrict__ kq_ws, const uint8_t* __restrict__ tp_ws,
                   const float* __restrict__ gb_ws, const float* init_state, float* __restrict__ y_raw,
                   float* final_state) {
  constexpr int NV = TC_NV;
  const int n = blockIdx.x, h = blockIdx.y, i0 = blockIdx.z * NV;
  const int hq = d.h_qk, hv = d.h_v, G = hv / hq, j = h / G;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int ts = cu ? cu[n] : 0, te = cu ? cu[n + 1] : d.total_tokens;
  const int nchunks = te > ts ? (te - ts + CH - 1) / CH : 0;
  const int gc0 = seq_chunk0[n];
  extern __shared__ __align__(128) uint8_t sm[];
  // small operand tiles first, then the two input stages
  uint8_t* s_hi = sm;
  uint8_t* s_lo = s_hi + PB_S_TILE;
  uint8_t* r_hi = s_lo + PB_S_TILE;  // R, then U-tilde
  uint8_t* r_lo = r_hi + PB_R_TILE;
  uint8_t* const stage0 = r_lo + PB_R_TILE;
  uint8_t* stage[2] = {stage0, stage0 + PBStage::BYTES};
  __shared__ uint64_t mbar_ld[2];
  __shared__ uint64_t mbar_mma;
  __shared__ uint32_t tslot;
  __shared__ int s_abort;

  // state slice S[i0 + i][j'] as S^T rows: thread tid owns key component j' = tid
  float S[NV];
  const size_t sbase = (((size_t)n * hv + h) * D + i0) * D;
#pragma unroll
  for (int i = 0; i < NV; ++i) S[i] = init_state ? init_state[sbase + (size_t)i * D + tid] : 0.0f;

  if (tid == 0) {
    s_abort = 0;
    tc::mbar_init(tc::smem_u32(&mbar_ld[0]), 1);
    tc::mbar_init(tc::smem_u32(&mbar_ld[1]), 1);
    tc::mbar_init(tc::smem_u32(&mbar_mma), 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(&tslot), 128);
    tc::tmem_relinquish();
  }
  auto issue_load = [&](int c, int st) {
    const size_t gc = (size_t)gc0 + c;
    const uint32_t bar = tc::smem_u32(&mbar_ld[st]);
    tc::mbar_arrive_expect_tx(bar, PBStage::BYTES);
    const uint32_t dst = tc::smem_u32(stage[st]);
    tc::bulk_g2s(dst + PBStage::KQ, kq_ws + (gc * hq + j) * KQ_BYTES, KQ_BYTES, bar);
    tc::bulk_g2s(dst + PBStage::TP, tp_ws + (gc * hv + h) * TP_BYTES, TP_BYTES, bar);
    tc::bulk_g2s(dst + PBStage::GB, gb_ws + (gc * hv + h) * GB_FLOATS, GB_FLOATS * 4, bar);
  };
  // S^T operand: thread j' writes its row (K index j', N = nv values) into the MN-major tile
  auto write_s_tile = [&]() {
#pragma unroll
    for (int nb = 0; nb < NV / 8; ++nb) {
      uint4 hi, lo;
      tc::split8(S + nb * 8, hi, lo);
      const uint32_t off = mnmaj(tid, nb, 128);
      *reinterpret_cast<uint4*>(s_hi + off) = hi;
      *reinterpret_cast<uint4*>(s_lo + off) = lo;
    }
  };
  write_s_tile();
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = tslot;
  const uint32_t t_a = tbase, t_cd = tbase + NV, t_e = tbase + 2 * NV;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  if (tid == 0 && nchunks > 0) issue_load(0, 0);

  // conv taps of this slice's value channels (used by warps 0..1)
  const size_t vch0 = (size_t)2 * hq * D + (size_t)h * D + i0;
  uint32_t ph_ld[2] = {0, 0}, ph_mma = 0;
  bool aborted = false;
  for (int c = 0; c < nchunks && !aborted; ++c) {
    const int st = c & 1;
    const int t0 = ts + c * CH, L = min(CH, te - t0);
    const uint8_t* sg = stage[st];
    // prefetch the next chunk into the other stage (its last reader finished last chunk)
    if (tid == 0 && c + 1 < nchunks) issue_load(c + 1, st ^ 1);
    // value rows of this chunk for R (warps 0..1: thread = token row t), conv + SiLU
    float vc[NV];
    const int t = tid & 63;
    if (warp < 2) {
#pragma unroll
      for (int i = 0; i < NV; ++i) vc[i] = 0.0f;
      if (t < L) {
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) {
          const long tg = (long)t0 + t - 3 + tap;
          if (tg < ts) continue;
          const uint16_t* row = v + ((size_t)tg * hv + h) * D + i0;
#pragma unroll
          for (int q4 = 0; q4 < NV / 8; ++q4) {
            const uint4 u = *reinterpret_cast<const uint4*>(row + q4 * 8);
            const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const int i = q4 * 8 + p * 2;
              vc[i] = fmaf(conv_w[(vch0 + i) * 4 + tap], bf2f(wds[p] & 0xffffu), vc[i]);
              vc[i + 1] = fmaf(conv_w[(vch0 + i + 1) * 4 + tap], bf2f(wds[p] >> 16), vc[i + 1]);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < NV; ++i) vc[i] = silu_f(vc[i]);
      }
    }
    if (!tc::mbar_wait(tc::smem_u32(&mbar_ld[st]), ph_ld[st])) { s_abort = 1; atomicExch(&g_gdn_status, -7); }
    ph_ld[st] ^= 1;
    const float* gsm = reinterpret_cast<const float*>(sg + PBStage::GB);
    const float gL = gsm[L - 1];
    // ---- round 1: [K S^T ; Q S^T] = [K;Q] (128 x 128) x S^T (K = 128, N = nv) -------------
    __syncthreads();
    if (s_abort) { aborted = true; break; }
    if (tid == 0) {
      tc::tc_fence_after();
      constexpr uint32_t idesc = tc::idesc_bf16(128, NV, 0, 1);
      const uint32_t a0[2] = {tc::smem_u32(sg + PBStage::KQ), tc::smem_u32(sg + PBStage::KQ + KQ_TILE)};
      const uint32_t b0[2] = {tc::smem_u32(s_hi), tc::smem_u32(s_lo)};
      for (int ks = 0; ks < 8; ++ks)
        for (int term = 0; term < 3; ++term) {
          const int ai = term == 2, bi = term == 1;
          tc::umma_bf16(t_a, tc::sdesc(a0[ai] + ks * 2 * LBO128, LBO128, 128),
                        tc::sdesc(b0[bi] + ks * 256, 128, 16 * 128), idesc, (ks | term) != 0);
        }
      tc::umma_commit(tc::smem_u32(&mbar_mma));
    }
    if (!tc::mbar_wait(tc::smem_u32(&mbar_mma), ph_mma)) { s_abort = 1; atomicExch(&g_gdn_status, -7); }
    ph_mma ^= 1;
    tc::tc_fence_after();
    float qs[NV];  // warps 2..3: e^{gamma_t} (Q S^T)[t][:]
    {
      uint32_t r[32];
      tc::tmem_ld32(t_a + lane_off, r);
      tc::tmem_wait_ld();
      if (warp < 2) {  // R[t][i] = beta_t (v[t][i] - e^{gamma_t} (K S^T)[t][i])
        const float eg = t < L ? expf(gsm[t]) : 0.0f, bt = t < L ? gsm[64 + t] : 0.0f;
        float rr[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) rr[i] = bt * (vc[i] - eg * __uint_as_float(r[i]));
#pragma unroll
        for (int nb = 0; nb < NV / 8; ++nb) {
          uint4 hi, lo;
          tc::split8(rr + nb * 8, hi, lo);
          const uint32_t off = mnmaj(t, nb, 64);
          *reinterpret_cast<uint4*>(r_hi + off) = hi;
          *reinterpret_cast<uint4*>(r_lo + off) = lo;
        }
      } else {
        const float eg = t < L ? expf(gsm[t]) : 0.0f;
#pragma unroll
        for (int i = 0; i < NV; ++i) qs[i] = eg * __uint_as_float(r[i]);
      }
    }
    tc::fence_proxy_async();
    tc::tc_fence_before();
    __syncthreads();
    if (s_abort) { aborted = true; break; }
    // ---- round 2: [U ; (M o QK^T) U] = [T;P] (128 x 64) x R (K = 64, N = nv) ----------------
    if (tid == 0) {
      tc::tc_fence_after();
      constexpr uint32_t idesc = tc::idesc_bf16(128, NV, 0, 1);
      const uint32_t a0[2] = {tc::smem_u32(sg + PBStage::TP), tc::smem_u32(sg + PBStage::TP + TP_TILE)};
      const uint32_t b0[2] = {tc::smem_u32(r_hi), tc::smem_u32(r_lo)};
      for (int ks = 0; ks < 4; ++ks)
        for (int term = 0; term < 3; ++term) {
          const int ai = term == 2, bi = term == 1;
          tc::umma_bf16(t_cd, tc::sdesc(a0[ai] + ks * 2 * LBO128, LBO128, 128),
                        tc::sdesc(b0[bi] + ks * 256, 128, 8 * 128), idesc, (ks | term) != 0);
        }
      tc::umma_commit(tc::smem_u32(&mbar_mma));
    }
    if (!tc::mbar_wait(tc::smem_u32(&mbar_mma), ph_mma)) { s_abort = 1; atomicExch(&g_gdn_status, -7); }
    ph_mma ^= 1;
    tc::tc_fence_after();
    {
      uint32_t r[32];
      tc::tmem_ld32(t_cd + lane_off, r);
      tc::tmem_wait_ld();
      if (warp < 2) {  // U-tilde[t][i] = e^{gamma_L - gamma_t} U[t][i]
        const float f = t < L ? expf(gL - gsm[t]) : 0.0f;
        float uu[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) uu[i] = f * __uint_as_float(r[i]);
#pragma unroll
        for (int nb = 0; nb < NV / 8; ++nb) {
          uint4 hi, lo;
          tc::split8(uu + nb * 8, hi, lo);
          const uint32_t off = mnmaj(t, nb, 64);
          *reinterpret_cast<uint4*>(r_hi + off) = hi;
          *reinterpret_cast<uint4*>(r_lo + off) = lo;
        }
      } else if (t < L) {  // Y = e^gamma Q S^T + (M o QK^T) U
        float* yr = y_raw + ((size_t)(t0 + t) * hv + h) * D + i0;
#pragma unroll
        for (int q4 = 0; q4 < NV / 4; ++q4) {
          float4 o;
          o.x = qs[q4 * 4 + 0] + __uint_as_float(r[q4 * 4 + 0]);
          o.y = qs[q4 * 4 + 1] + __uint_as_float(r[q4 * 4 + 1]);
          o.z = qs[q4 * 4 + 2] + __uint_as_float(r[q4 * 4 + 2]);
          o.w = qs[q4 * 4 + 3] + __uint_as_float(r[q4 * 4 + 3]);
          *reinterpret_cast<float4*>(yr + q4 * 4) = o;
        }
      }
    }
    tc::fence_proxy_async();
    tc::tc_fence_before();
    __syncthreads();
    if (s_abort) { aborted = true; break; }
    // ---- round 3: K^T U-tilde: A = MN-major view of the K rows (M = 128 key comps, K = 64 tokens)
    if (tid == 0) {
      tc::tc_fence_after();
      constexpr uint32_t idesc = tc::idesc_bf16(128, NV, 1, 1);
      const uint32_t a0[2] = {tc::smem_u32(sg + PBStage::KQ), tc::smem_u32(sg + PBStage::KQ + KQ_TILE)};
      const uint32_t b0[2] = {tc::smem_u32(r_hi), tc::smem_u32(r_lo)};
      for (int ks = 0; ks < 4; ++ks)
        for (int term = 0; term < 3; ++term) {
          const int ai = term == 2, bi = term == 1;
          tc::umma_bf16(t_e, tc::sdesc(a0[ai] + ks * 256, 128, LBO128),
                        tc::sdesc(b0[bi] + ks * 256, 128, 8 * 128), idesc, (ks | term) != 0);
        }
      tc::umma_commit(tc::smem_u32(&mbar_mma));
    }
    if (!tc::mbar_wait(tc::smem_u32(&mbar_mma), ph_mma)) { s_abort = 1; atomicExch(&g_gdn_status, -7); }
    ph_mma ^= 1;
    tc::tc_fence_after();
    {
      uint32_t r[32];
      tc::tmem_ld32(t_e + lane_off, r);
      tc::tmem_wait_ld();
      const float eL = expf(gL);
#pragma unroll
      for (int i = 0; i < NV; ++i) S[i] = fmaf(eL, S[i], __uint_as_float(r[i]));
    }
    write_s_tile();
    tc::fence_proxy_async();
    tc::tc_fence_before();
    __syncthreads();
    if (s_abort) { aborted = true; break; }
  }
  // final state slice (thread j' writes column j' of rows i0 .. i0 + nv)
  if (!aborted) {
#pragma unroll
    for (int i = 0; i < NV; ++i) final_state[sbase + (size_t)i * D + tid] = S[i];
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 128);
}

}  // namespace gdn
