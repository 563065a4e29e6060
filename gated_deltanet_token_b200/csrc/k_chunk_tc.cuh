// k_chunk_tc.cuh -- chunked gated delta rule on tcgen05 tensor cores (bf16-input path).
//
// Same chunk algebra as k_chunk_simt.cuh (an exact rewrite of the six steps of the
// "Qwen3-Next 80B-A3B" field guide, §02; the state carry is the chunk-loop update of the
// "Qwen3.8-Flash-Next" model notes in column-vector form), regrouped so that every
// contraction is an M = 128 tcgen05 MMA:
//
//   R   = V - diag(e^gamma) K S^T                           [U = T diag(beta) R, T = (I + A)^-1]
//   [U ; M o QK^T U] = [T ; P] diag(beta) R,  P = (M o QK^T) T   (one MMA, 128 x nv x 64)
//   Y   = diag(e^gamma) Q S^T + (M o QK^T) U
//   S^T <- e^{gamma_L} S^T + K^T diag(e^{gamma_L - gamma}) U
//   [K S^T ; Q S^T] = [K ; Q] S^T                            (one MMA, 128 x nv x 128)
//
// Every tensor-core product is taken in three bf16 terms, a_hi b_hi + a_hi b_lo + a_lo b_hi,
// with x = hi + lo the bf16 split of an fp32 value: plain bf16 operands lose ~2^-9 per
// element, which the scale-invariant output norm amplifies on tokens with a small y_raw;
// the split keeps the products at ~2^-17 relative error.
//
// Phase A (k_chunkprep_tc, parallel over chunks x QK heads), prologue included: the chunk's
// raw q, k, v rows by tensor copy; conv + SiLU of q, k, v and the L2 norm of q and k; the
// [K;Q] hi/lo operand tile of each (chunk, QK head) and v as fp32 slices for phase B;
// [K;Q] K^T on tcgen05; for both value heads of a pair at once: gates, gamma, A, M o QK^T,
// T = (I + A)^-1 (blocked 16 x 16 forward substitution), P = (M o QK^T) T, and the [T;P]
// hi/lo tiles with beta folded into their columns.
// Phase B (k_chunkscan_tc, sequential over one sequence's chunks, parallel over value
// heads and 32-row slices of the state): the three MMA rounds above per chunk, with the
// next chunk's tiles bulk-copied into a second stage while the current one computes, and
// (by default) the gated output norm fused in.
#pragma once
#include <cuda.h>

#include "gdn_common.cuh"
#include "tc_ptx.cuh"

namespace gdn {

constexpr int TC_NV = 32;                            // state rows (value components) per phase-B CTA
constexpr uint32_t KQ_TILE = 128 * 128 * 2;          // one bf16 tile of [K;Q] (hi or lo): 32 KB
constexpr uint32_t KQ_BYTES = 2 * KQ_TILE;           // per (chunk, QK head)
constexpr uint32_t TP_TILE = 128 * 64 * 2;           // one bf16 tile of [T;P]: 16 KB
constexpr uint32_t TP_BYTES = 2 * TP_TILE;           // per (chunk, value head)
constexpr uint32_t GB_FLOATS = 128;                  // gamma[64], gamma_L - gamma[64] per (chunk, value head)
constexpr uint32_t VS_SLICE = 64 * TC_NV * 4;        // v after conv + SiLU (fp32), one 32-column slice: 8 KB
constexpr uint32_t VS_BYTES = 4 * VS_SLICE;          // per (chunk, value head)
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
// view), B MN-major K=64 N=32; case 4: as case 1 with A copied into TMEM first (tcgen05.cp)
// and read from there by the MMA; case 5: M = 64 from rows 64..127 of the 128-row A tile, B
// MN-major K=128 N=32, the result read from TMEM lanes 0..15 of each 32-lane quarter.
// out[0] = max |D - ref|, out[1] = max |ref|.
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
  constexpr int K = (CASE == 0 || CASE == 1 || CASE == 4 || CASE == 5) ? 128 : 64;
  constexpr int M = CASE == 5 ? 64 : 128;
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
  // case 5: logical row m of A is physical row 64 + m
  auto Aval = [&](int m, int k) {
    return CASE == 3 ? st_val(k * 128 + m, 11u) : st_val((m + (CASE == 5 ? 64 : 0)) * 1024 + k, 1u + CASE % 4);
  };
  auto Bval = [&](int k, int n) { return CASE == 0 ? Aval(n, k) : st_val(k * 64 + n, 7u + CASE % 4); };
  // physical A tile (K-major, 128 rows): case 3 stores X[s][j] = A[j][s] at (r = s, k = j)
  for (int idx = tid; idx < ROWS_A * a_cols; idx += 128) {
    const int r = idx / a_cols, c = idx % a_cols;
    float v = CASE == 3 ? (r < 64 ? Aval(c, r) : 0.0f) : CASE == 5 ? st_val(r * 1024 + c, 2u) : Aval(r, c);
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
    tc::tmem_alloc(tc::smem_u32(&tslot), CASE == 4 ? 256 : 64);
    tc::tmem_relinquish();
  }
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = tslot;
  bool ok = true;
  if (CASE == 4) {  // A hi -> TMEM columns 64.., A lo -> 128.., then read by the MMA from there
    if (tid == 0) {
      for (int ks = 0; ks < K / 16; ++ks) {
        tc::tmem_cp_128x256b(tbase + 64 + ks * 8, tc::sdesc(tc::smem_u32(Ahi) + ks * 2 * LBO128, LBO128, 128));
        tc::tmem_cp_128x256b(tbase + 128 + ks * 8, tc::sdesc(tc::smem_u32(Alo) + ks * 2 * LBO128, LBO128, 128));
      }
      tc::umma_commit(tc::smem_u32(&mbar));
    }
    ok = tc::mbar_wait(tc::smem_u32(&mbar), 0);
    tc::tc_fence_after();
  }
  if (tid == 0 && CASE == 4 && ok) {
    constexpr uint32_t idesc = tc::idesc_bf16(128, N, 0, 1);
    const uint32_t b0[2] = {tc::smem_u32(Bhi), tc::smem_u32(Blo)};
    for (int ks = 0; ks < K / 16; ++ks)
      for (int term = 0; term < 3; ++term) {
        const uint32_t at = tbase + (term == 2 ? 128 : 64) + ks * 8;
        const uint64_t bd = tc::sdesc(b0[term == 1] + ks * 2 * 128, 128, (K / 8) * 128);
        tc::umma_bf16_ts(tbase, at, bd, idesc, (ks | term) != 0);
      }
    tc::umma_commit(tc::smem_u32(&mbar));
  }
  if (tid == 0 && CASE != 4) {
    constexpr uint32_t idesc = tc::idesc_bf16(M, N, CASE == 3 ? 1 : 0, CASE == 0 ? 0 : 1);
    const uint32_t a0[2] = {tc::smem_u32(Ahi), tc::smem_u32(Alo)};
    const uint32_t b0[2] = {CASE == 0 ? tc::smem_u32(Ahi) : tc::smem_u32(Bhi),
                            CASE == 0 ? tc::smem_u32(Alo) : tc::smem_u32(Blo)};
    // A: K-major (LBO 2048, SBO 128) or, case 3, MN-major view (SBO 2048, LBO 128).
    const uint32_t a_lbo = CASE == 3 ? 128 : LBO128, a_sbo = CASE == 3 ? LBO128 : 128;
    const uint32_t b_lbo = CASE == 0 ? LBO128 : 128, b_sbo = CASE == 0 ? 128 : (K / 8) * 128;
    for (int ks = 0; ks < K / 16; ++ks) {
      for (int term = 0; term < 3; ++term) {
        const int ai = term == 2 ? 1 : 0, bi = term == 1 ? 1 : 0;
        const uint64_t ad = tc::sdesc(a0[ai] + ks * 2 * a_lbo + (CASE == 5 ? 8 * 128 : 0), a_lbo, a_sbo);
        const uint64_t bd = tc::sdesc(b0[bi] + ks * 2 * b_lbo, b_lbo, b_sbo);
        tc::umma_bf16(tbase, ad, bd, idesc, (ks | term) != 0);
      }
    }
    tc::umma_commit(tc::smem_u32(&mbar));
  }
  ok = ok && tc::mbar_wait(tc::smem_u32(&mbar), CASE == 4 ? 1 : 0);
  tc::tc_fence_after();
  const int m = CASE == 5 ? warp * 16 + (lane & 15) : warp * 32 + lane;  // row held by this lane
  const bool holds = CASE != 5 || lane < 16;  // M = 64: lanes 16..31 of a quarter hold no row
  float err = 0.0f, mag = 0.0f;
  if (ok) {
    for (int n0 = 0; n0 < N; n0 += 32) {
      uint32_t r[32];
      tc::tmem_ld32(tbase + ((uint32_t)(warp * 32) << 16) + n0, r);  // the whole warp loads
      tc::tmem_wait_ld();
      for (int c = 0; c < 32 && holds; ++c) {
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
  if (warp == 0) tc::tmem_dealloc(tbase, CASE == 4 ? 256 : 64);
}

// ======================================================================================
// Diagnostic of the bounded waits (gdn_selftest_wait_timeout): one CTA holds tensor memory and
// waits on an mbarrier that nothing completes -- no copy and no MMA is ever issued -- with the
// same bounded wait the prefill kernels use.  The wait runs out, the timeout is recorded in the
// device status word and the CTA frees its tensor memory and returns.
// ======================================================================================
__global__ void __launch_bounds__(128) k_selftest_wait_timeout() {
  __shared__ uint64_t mbar;
  __shared__ uint32_t tslot;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    tc::mbar_init(tc::smem_u32(&mbar), 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(&tslot), 32);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = tslot;
  // warp-uniform, as the prefill kernels take it ahead of their warp-collective TMEM loads
  const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&mbar), 0));
  if (!ok && threadIdx.x == 0) atomicExch(&g_gdn_status, -7);
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 32);
}

// ======================================================================================
// Phase A
// ======================================================================================
constexpr int PA_P = 68;  // pitch (floats) of the fp32 64 x 64 matrices of phase A
constexpr uint32_t PA_MAT = 64 * PA_P * 4;
// [0, 64K): the [K;Q] tile (hi | lo).  Once [K;Q]K^T is in TMEM the tile is dead and the
// region holds the P operands, [Mq_a; Mq_b] (K-major, 128 x 64) hi | lo at [0, 32K) and
// [T_a | T_b] (MN-major, K = 64, N = 128) hi | lo at [32K, 64K); the fp32 A matrices of both
// heads of the pair alias [32K, 32K + 2 PA_MAT) until T is known.  Then the fp32 T matrices
// of the pair and the gates.
constexpr uint32_t PA_OFF_PA = 0;
constexpr uint32_t PA_OFF_PB = 32768;
constexpr uint32_t PA_OFF_A = 32768;
constexpr uint32_t PA_OFF_T = PA_OFF_A + 2 * PA_MAT;
constexpr uint32_t PA_OFF_G = PA_OFF_T + 2 * PA_MAT;
constexpr uint32_t PA_OFF_W = PA_OFF_G + 2 * 64 * 8 + 2 * 64 * 4;  // [16 half-warps][16 rows] float4 scratch
constexpr size_t PA_TC_SMEM = PA_OFF_W + 16 * 16 * 16;
static_assert(PA_OFF_T >= KQ_BYTES, "T and the gates lie past the [K;Q] tile");
static_assert(PA_TC_SMEM <= 113 * 1024, "two phase-A CTAs per SM");

// Raw rows of one chunk with its conv history (tokens t0 - 3 .. t0 + 63), as the tensor
// copies land them: [row][heads][128] bf16.  q and k of the QK head (one head each) and, later,
// a value-head pair (two heads) share the space of the T matrices, which the solve fills only
// after the raw rows have been consumed; the conv taps of two heads use the solve's scratch.
constexpr int PF_ROWS = CH + 3;
constexpr uint32_t PF_HEAD_BYTES = PF_ROWS * D * 2;  // one head's raw rows: 17,152 B
constexpr uint32_t PF_OFF_QRAW = PA_OFF_T;
constexpr uint32_t PF_OFF_KRAW = PA_OFF_T + PF_HEAD_BYTES;
constexpr uint32_t PF_OFF_VRAW = PA_OFF_T;
constexpr uint32_t PF_OFF_TAPS = PA_OFF_W;
static_assert(PA_OFF_T + 2 * PF_HEAD_BYTES <= PA_OFF_G, "raw rows fit in the T matrices' space");
static_assert(PA_OFF_W + 2 * D * 16 <= PA_TC_SMEM, "conv taps of two heads fit in the solve scratch");
static_assert(PF_OFF_QRAW % 128 == 0 && PF_OFF_KRAW % 128 == 0 && PF_OFF_TAPS % 16 == 0,
              "tensor-copy destinations are 128-byte aligned");
static_assert(PF_ROWS <= 256, "tensor-copy box limit");

// One CTA per (QK head j, chunk), prologue included: the chunk's raw q and k rows (with three
// rows of conv history) arrive by tensor copy; the width-4 causal conv, SiLU and L2 norm
// ("Qwen3.8-Flash-Next" technical report, Fig. 2; field guide §02) build the [K;Q] hi/lo
// operand tile in shared memory, which is stored once for phase B.  Then, for the value heads
// of QK head j in pairs (a, b), both heads of a pair at once: conv + SiLU of v (fp32 slices for
// phase B), the gates, A, M o QK^T, T = (I + A)^-1 and P = (M o QK^T) T.  Field guide §02
// defines the per-token steps these chunk quantities regroup.
__global__ void __launch_bounds__(256, 2)
    k_chunkprep_tc(Dims d, const ChunkEntry* __restrict__ tab, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const float* __restrict__ conv_w, const float* __restrict__ a,
                   const float* __restrict__ b, const float* __restrict__ A_log,
                   const float* __restrict__ dt_bias, uint8_t* __restrict__ kq_ws, float* __restrict__ vs_ws,
                   uint8_t* __restrict__ tp_ws, float* __restrict__ gb_ws) {
  tc::grid_dep_wait();  // all earlier work on the stream (the inputs, the last call's use of the workspace) is done
  tc::grid_dep_launch_dependents();
  // head-fastest grid, chunks from the last: the early chunks' tiles, written last, are still in
  // L2 when phase B starts on them
  const int chunk = gridDim.y - 1 - blockIdx.y;
  const ChunkEntry e = chunk_entry(tab, d.total_tokens, chunk);
  if (e.len == 0) return;
  const int j = blockIdx.x, hq = d.h_qk, hv = d.h_v, G = hv / hq, L = e.len;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* kq_hi = sm;
  uint8_t* kq_lo = sm + KQ_TILE;
  uint8_t* pa_hi = sm + PA_OFF_PA;  // [Mq_a; Mq_b] operand (aliases the [K;Q] tile)
  uint8_t* pa_lo = pa_hi + 16384;
  uint8_t* pb_hi = sm + PA_OFF_PB;  // [T_a | T_b] operand
  uint8_t* pb_lo = pb_hi + 16384;
  float* Am = reinterpret_cast<float*>(sm + PA_OFF_A);  // [2][64][PA_P]
  float* Tm = reinterpret_cast<float*>(sm + PA_OFF_T);  // [2][64][PA_P]
  float2* gs = reinterpret_cast<float2*>(sm + PA_OFF_G);               // [2][64] gamma as hi + lo
  float* bs = reinterpret_cast<float*>(sm + PA_OFF_G + 2 * 64 * 8);   // [2][64] beta
  float4* wsc = reinterpret_cast<float4*>(sm + PA_OFF_W) + (tid >> 4) * 16;  // this half-warp's rows
  const float4* taps = reinterpret_cast<const float4*>(sm + PF_OFF_TAPS);   // [2][128] conv taps
  __shared__ uint64_t mbar;     // MMA completions
  __shared__ uint64_t mbar_ld;  // tensor / bulk copies of raw rows and taps
  __shared__ uint32_t tslot;
  __shared__ int s_abort;

  if ((tc::smem_u32(sm) & 127u) != 0) {  // tensor copies need 128-byte aligned destinations
    if (tid == 0) atomicExch(&g_gdn_status, -6);
    return;
  }
  if (tid == 0) {
    s_abort = 0;
    tc::mbar_init(tc::smem_u32(&mbar), 1);
    tc::mbar_init(tc::smem_u32(&mbar_ld), 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(&tslot), 256);  // cols 0..63: [K;Q]K^T, 128..255: P pair
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = tslot;
  // (thread 0) raw rows of two heads of one stream and their conv taps into the raw space
  int ld_issued = 0, ld_waited = 0;  // armings of mbar_ld (thread 0) and waits on it (every thread)
  auto issue_raw = [&](const CUtensorMap* tm0, int head0, const CUtensorMap* tm1, int head1, int ch0, int ch1,
                       uint32_t box_bytes) {
    const uint32_t bar = tc::smem_u32(&mbar_ld);
    ++ld_issued;
    tc::mbar_arrive_expect_tx(bar, box_bytes + (ch1 >= 0 ? 2u : 1u) * D * 16);
    tc::tma_load_3d(tc::smem_u32(sm + PF_OFF_QRAW), tm0, 0, head0, e.t0 - 3, bar);
    if (tm1) tc::tma_load_3d(tc::smem_u32(sm + PF_OFF_KRAW), tm1, 0, head1, e.t0 - 3, bar);
    tc::bulk_g2s(tc::smem_u32(sm + PF_OFF_TAPS), conv_w + (size_t)ch0 * 4, D * 16, bar);
    if (ch1 >= 0) tc::bulk_g2s(tc::smem_u32(sm + PF_OFF_TAPS) + D * 16, conv_w + (size_t)ch1 * 4, D * 16, bar);
  };
  // the value-head pair starting at head index g0 of QK head j (the second head's taps only if
  // it exists: its box rows past the tensor read as zeros)
  auto issue_v = [&](int g0) {
    const int h0 = j * G + g0;
    issue_raw(&tm_v, h0, nullptr, 0, 2 * hq * D + h0 * D, g0 + 1 < G ? 2 * hq * D + (h0 + 1) * D : -1,
              2 * PF_HEAD_BYTES);
  };
  if (tid == 0) issue_raw(&tm_q, j, &tm_k, j, j * D, (hq + j) * D, 2 * PF_HEAD_BYTES);
  uint32_t ld_phase = 0, mma_phase = 0;
  // raw row rr holds token t0 - 3 + rr: usable if inside the chunk and the sequence
  auto row_ok = [&](int rr) {
    const int tcr = rr - 3;
    return tcr < L && e.t0 + tcr >= e.seq_start;
  };
  bool aborted = false;
  for (int ga = 0; ga < G; ga += 2) {
    const int gpair[2] = {ga, ga + 1 < G ? ga + 1 : ga};
    if (warp < 2) {  // gates and gamma of the pair: warp 0 head a, warp 1 head b
      const int h = j * G + gpair[warp];
      // gamma is a prefix sum in fp64: a decay factor e^{gamma_t - gamma_s} is formed from the
      // difference of two prefixes, which in fp32 would lose ulp(|gamma|) -- about 2e-4 once a
      // few strong decays (g of several hundred) have accumulated in the chunk
      double g0 = 0.0, g1 = 0.0;
      float b0 = 0.0f, b1 = 0.0f;
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
        const double y0 = __shfl_up_sync(0xffffffffu, g0, o);
        const double y1 = __shfl_up_sync(0xffffffffu, g1, o);
        if (lane >= o) { g0 += y0; g1 += y1; }
      }
      g1 += __shfl_sync(0xffffffffu, g0, 31);
      const double gL = __shfl_sync(0xffffffffu, g1, 31);  // gamma at the chunk's end (padding adds 0)
      // gamma as an unevaluated float pair hi + lo (|lo| <= ulp(hi) / 2): a difference of two
      // prefixes, (hi_t - hi_s) + (lo_t - lo_s), then has a relative error of a few fp32 ulp of
      // the difference itself, whatever the size of gamma, and needs no fp64 arithmetic per element
      const float h0f = (float)g0, h1f = (float)g1;
      gs[warp * 64 + lane] = make_float2(h0f, (float)(g0 - (double)h0f));
      gs[warp * 64 + lane + 32] = make_float2(h1f, (float)(g1 - (double)h1f));
      bs[warp * 64 + lane] = b0; bs[warp * 64 + lane + 32] = b1;
      if (warp == 0 || gpair[1] != gpair[0]) {  // phase B's gates: gamma_t and gamma_L - gamma_t
        float* gbw = gb_ws + ((size_t)chunk * hv + h) * GB_FLOATS;
        gbw[lane] = (float)g0; gbw[lane + 32] = (float)g1;
        gbw[64 + lane] = (float)(gL - g0); gbw[96 + lane] = (float)(gL - g1);
      }
    }
    if (ga == 0) {
      // ---- prologue: conv + SiLU + L2 norm of k (warps 0..3) and q (warps 4..7) into the
      // [K;Q] tile; lane: token r = lane % 4 of a four-token block, channel groups g0 = lane / 4
      // and g0 + 8; the eight lanes of a token reduce its norm with three shuffles
      const bool okl = tc::mbar_wait(tc::smem_u32(&mbar_ld), ld_phase);
      ld_phase ^= 1;
      ++ld_waited;
      if (!okl) { s_abort = 1; atomicExch(&g_gdn_status, -7); }
      if (okl) {
        const int isq = warp >> 2;
        const uint16_t* raw = reinterpret_cast<const uint16_t*>(sm + (isq ? PF_OFF_QRAW : PF_OFF_KRAW));
        const float4* wsm = taps + (isq ? 0 : D);
        const int r = lane & 3, g0 = lane >> 2;
        const float scale = isq ? d.q_scale : 1.0f;
#pragma unroll 1
        for (int blk = (warp & 3) * 16; blk < (warp & 3) * 16 + 16; blk += 4) {
          const int t = blk + r;  // chunk-relative token; its taps read raw rows t .. t + 3
          float acc[2][8];
          bool okt[4];
#pragma unroll
          for (int tap = 0; tap < 4; ++tap) okt[tap] = row_ok(t + tap);
#pragma unroll
          for (int gi = 0; gi < 2; ++gi) {
            const int cg = (g0 + 8 * gi) * 8;
            uint32_t xw[4][4];
#pragma unroll
            for (int tap = 0; tap < 4; ++tap) {
              const uint4 x = okt[tap] ? *reinterpret_cast<const uint4*>(raw + (size_t)(t + tap) * D + cg)
                                       : make_uint4(0, 0, 0, 0);
              xw[tap][0] = x.x; xw[tap][1] = x.y; xw[tap][2] = x.z; xw[tap][3] = x.w;
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float4 w4 = wsm[cg + c];  // channel cg + c, taps 0..3
              float a_ = 0.0f;
#pragma unroll
              for (int tap = 0; tap < 4; ++tap)
                a_ = fmaf(comp(w4, tap), bf2f(c & 1 ? xw[tap][c >> 1] >> 16 : xw[tap][c >> 1] & 0xffffu), a_);
              acc[gi][c] = a_;
            }
          }
          float ss0 = 0.0f, ss1 = 0.0f;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            acc[0][c] = silu_fast(acc[0][c]);
            acc[1][c] = silu_fast(acc[1][c]);
            ss0 = fmaf(acc[0][c], acc[0][c], ss0);
            ss1 = fmaf(acc[1][c], acc[1][c], ss1);
          }
          float sst = ss0 + ss1;
          sst += __shfl_xor_sync(0xffffffffu, sst, 4);
          sst += __shfl_xor_sync(0xffffffffu, sst, 8);
          sst += __shfl_xor_sync(0xffffffffu, sst, 16);
          const float inv = t < L ? scale * rsqrtf(sst + d.l2_eps) : 0.0f;
          const int row = (isq ? 64 : 0) + t;
#pragma unroll
          for (int gi = 0; gi < 2; ++gi) {
            float x8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) x8[c] = acc[gi][c] * inv;
            uint4 hi, lo;
            tc::split8(x8, hi, lo);
            const uint32_t off = kmaj128(row, (g0 + 8 * gi) * 8);
            *reinterpret_cast<uint4*>(kq_hi + off) = hi;
            *reinterpret_cast<uint4*>(kq_lo + off) = lo;
          }
        }
      }
      tc::fence_proxy_async();  // the tile's generic stores, for the MMA and the bulk store
      tc::tc_fence_before();
      __syncthreads();          // the tile is complete and the raw q / k rows are consumed
      tc::tc_fence_after();
      if (tid == 0 && !s_abort) {
        // the tile for phase B, then the first value pair's raw rows into the freed raw space
        tc::bulk_s2g(kq_ws + ((size_t)chunk * hq + j) * KQ_BYTES, tc::smem_u32(sm), KQ_BYTES);
        tc::bulk_commit();
        issue_v(0);
        // [K;Q] K^T (the gates above overlapped the raw copies)
        constexpr uint32_t idesc = tc::idesc_bf16(128, 64, 0, 0);
        const uint64_t dd[2] = {tc::sdesc(tc::smem_u32(kq_hi), LBO128, 128), tc::sdesc(tc::smem_u32(kq_lo), LBO128, 128)};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
          for (int term = 0; term < 3; ++term) {
            const uint64_t o = (uint64_t)((ks * 2 * LBO128) >> 4);
            tc::umma_bf16(tbase, dd[term == 2] + o, dd[term == 1] + o, idesc, (ks | term) != 0);
          }
        tc::umma_commit(tc::smem_u32(&mbar));
      }
      if (!s_abort && !tc::mbar_wait(tc::smem_u32(&mbar), mma_phase)) { s_abort = 1; atomicExch(&g_gdn_status, -7); }
      mma_phase ^= 1;
      tc::tc_fence_after();
      // the A matrices below overwrite the tile's lo half: the bulk store must have read it
      if (tid == 0) tc::bulk_wait_read_all();
    }
    __syncthreads();
    aborted = s_abort != 0;
    if (aborted) break;
    // A (fp32) of both heads and the Mq rows of the P operand, straight from the [K;Q]K^T
    // accumulator: warp w reads TMEM lanes 32 (w % 4).. (rows 0..63 K K^T, 64..127 Q K^T),
    // columns 32 (w / 4) .. + 31.
    {
      const int q4 = warp & 3, cbk = (warp >> 2) * 32;
      const int t = (q4 * 32 + lane) & 63;
      uint32_t r[32];
      tc::tmem_ld32(tbase + ((uint32_t)(q4 * 32) << 16) + cbk, r);
      tc::tmem_wait_ld();
#pragma unroll 1
      for (int hp = 0; hp < 2; ++hp) {
        const float2* g_ = gs + hp * 64;
        const float2 gt = g_[t];
        // the block of columns cbk .. cbk + 31 lies wholly above the diagonal for rows 0..31
        // (warp-uniform): zeros, with no exponentials
        const bool upper = cbk > (q4 & 1) * 32;
        if (q4 < 2) {  // A[t][s] = beta_t e^{gamma_t - gamma_s} (k_t . k_s), s < t
          const float bt = bs[hp * 64 + t];
          float* Ah = Am + hp * (64 * PA_P);
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            float4 o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            float* op = &o.x;
            if (!upper) {
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int s_ = cbk + c4 * 4 + u;
                op[u] = s_ < t ? bt * __expf((gt.x - g_[s_].x) + (gt.y - g_[s_].y)) * __uint_as_float(r[c4 * 4 + u])
                               : 0.0f;
              }
            }
            *reinterpret_cast<float4*>(Ah + t * PA_P + cbk + c4 * 4) = o;
          }
        } else {  // Mq[t][s] = e^{gamma_t - gamma_s} (q_t . k_s), s <= t  (mask before exp)
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float mv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int s_ = cbk + c8 * 8 + u;
              mv[u] = (!upper && s_ <= t)
                          ? __expf((gt.x - g_[s_].x) + (gt.y - g_[s_].y)) * __uint_as_float(r[c8 * 8 + u])
                          : 0.0f;
            }
            uint4 hi, lo;
            tc::split8(mv, hi, lo);
            *reinterpret_cast<uint4*>(pa_hi + kmaj128(hp * 64 + t, cbk + c8 * 8)) = hi;
            *reinterpret_cast<uint4*>(pa_lo + kmaj128(hp * 64 + t, cbk + c8 * 8)) = lo;
          }
        }
      }
    }
    __syncthreads();
    // ---- v of the pair: conv + SiLU as four contiguous 32-column fp32 slices per head for
    // phase B.  Warp w: head w / 4 of the pair, tokens 16 (w % 4) .. + 15 in two blocks of
    // eight (raw rows blk .. blk + 10); lane: channels 4 lane .. 4 lane + 3.  Rows past the
    // chunk's length are written as zeros.
    {
      const bool okv = tc::mbar_wait(tc::smem_u32(&mbar_ld), ld_phase);
      ld_phase ^= 1;
      ++ld_waited;
      if (!okv) { s_abort = 1; atomicExch(&g_gdn_status, -7); }
      const int hp = warp >> 2;
      if (okv && (hp == 0 || gpair[1] != gpair[0])) {
        const int h = j * G + gpair[hp], c0 = lane * 4;
        const uint16_t* hrow = reinterpret_cast<const uint16_t*>(sm + PF_OFF_VRAW) + hp * D;  // row stride 2 D
        float wv[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float4 t4 = taps[hp * D + c0 + c];
          wv[c][0] = t4.x; wv[c][1] = t4.y; wv[c][2] = t4.z; wv[c][3] = t4.w;
        }
        float* out = vs_ws + ((size_t)chunk * hv + h) * (VS_BYTES / 4) + (size_t)(c0 / TC_NV) * (VS_SLICE / 4) +
                     (c0 % TC_NV);
#pragma unroll 1
        for (int blk = (warp & 3) * 16; blk < (warp & 3) * 16 + 16; blk += 8) {
          uint2 x[11];  // raw bf16 of the 4 channels, rows blk .. blk + 10 (tokens blk - 3 .. blk + 7)
#pragma unroll
          for (int p = 0; p < 11; ++p)
            x[p] = row_ok(blk + p) ? *reinterpret_cast<const uint2*>(hrow + (size_t)(blk + p) * 2 * D + c0)
                                   : make_uint2(0, 0);
          auto xv = [&](int p, int c) {
            const uint32_t wd = c < 2 ? x[p].x : x[p].y;
            return bf2f(c & 1 ? wd >> 16 : wd & 0xffffu);
          };
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int t = blk + i;
            float r4[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float acc = fmaf(wv[c][3], xv(i + 3, c),
                                     fmaf(wv[c][2], xv(i + 2, c), fmaf(wv[c][1], xv(i + 1, c), wv[c][0] * xv(i, c))));
              r4[c] = t < L ? silu_fast(acc) : 0.0f;
            }
            *reinterpret_cast<float4*>(out + t * TC_NV) = make_float4(r4[0], r4[1], r4[2], r4[3]);
          }
        }
      }
    }
    __syncthreads();  // the raw v rows and taps are consumed before the solve writes over them
    // T = (I + A)^-1 by 16 x 16 blocks: diagonal blocks by forward substitution (thread =
    // head, block, column; rows of A read as float4) ...
    if (tid < 128) {
      const int hp = tid >> 6, blk = (tid >> 4) & 3, c = tid & 15, o = blk * 16;
      const float* Ab = Am + hp * (64 * PA_P) + o * PA_P + o;
      float* Tb = Tm + hp * (64 * PA_P) + o * PA_P + o;
      float x[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        float ar[16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float4 a4 = *reinterpret_cast<const float4*>(Ab + t * PA_P + q4 * 4);
          ar[q4 * 4 + 0] = a4.x; ar[q4 * 4 + 1] = a4.y; ar[q4 * 4 + 2] = a4.z; ar[q4 * 4 + 3] = a4.w;
        }
        float v = (t == c) ? 1.0f : 0.0f;
#pragma unroll
        for (int r = 0; r < t; ++r) v = fmaf(-ar[r], x[r], v);
        x[t] = v;
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) Tb[t * PA_P + c] = x[t];
    }
    __syncthreads();
    // ... then by distance: T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj.  Item = (head, block
    // column bj, column quad, row rr); the 16 rows of a quad sit in one half-warp and share the
    // rows of W = sum_k A_ik T_kj through shared memory.  Blocks above the diagonal are never
    // read.
    for (int dist = 1; dist < 4; ++dist) {
      const int per_head = (4 - dist) * 64;
      for (int g = tid; g < 2 * per_head; g += 256) {  // warp-uniform: per_head is a multiple of 64
        const int hp = g >= per_head, i = g - hp * per_head;
        const float* Ah = Am + hp * (64 * PA_P);
        float* Th = Tm + hp * (64 * PA_P);
        const int rr = i & 15, cq = ((i >> 4) & 3) * 4, bj = i >> 6, bi = bj + dist;
        const int ti = bi * 16 + rr, tj = bj * 16 + cq;
        float4 wv = make_float4(0, 0, 0, 0);
        for (int kk = bj * 16; kk < bi * 16; kk += 4) {
          const float4 a4 = *reinterpret_cast<const float4*>(Ah + ti * PA_P + kk);
          const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float4 tv = *reinterpret_cast<const float4*>(Th + (kk + u) * PA_P + tj);
            wv.x = fmaf(av[u], tv.x, wv.x); wv.y = fmaf(av[u], tv.y, wv.y);
            wv.z = fmaf(av[u], tv.z, wv.z); wv.w = fmaf(av[u], tv.w, wv.w);
          }
        }
        float4 trow[4];  // T_ii row rr
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) trow[q4] = *reinterpret_cast<const float4*>(Th + ti * PA_P + bi * 16 + q4 * 4);
        wsc[rr] = wv;
        __syncwarp();
        float4 res = make_float4(0, 0, 0, 0);
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float tv = m <= rr ? comp(trow[m >> 2], m & 3) : 0.0f;
          const float4 w = wsc[m];
          res.x = fmaf(-tv, w.x, res.x); res.y = fmaf(-tv, w.y, res.y);
          res.z = fmaf(-tv, w.z, res.z); res.w = fmaf(-tv, w.w, res.w);
        }
        __syncwarp();  // the rows are read before the next item of this half-warp writes them
        *reinterpret_cast<float4*>(Th + ti * PA_P + tj) = res;
      }
      __syncthreads();
    }
    // T diag(beta) of both heads as columns hp * 64 .. of the MN-major B operand of P (over the
    // dead A matrices), and the T diag(beta) rows of each head's [T;P] output tile (K-major,
    // straight to the workspace); blocks above the diagonal are zeros.  With beta folded in
    // here, phase B forms R = V - diag(e^gamma) K S^T and [T;P] diag(beta) R gives U and
    // (M o QK^T) U.
    for (int it = tid; it < 2 * 64 * 8; it += 256) {
      const int hp = it >> 9, r = it & 63, s0 = ((it >> 6) & 7) * 8;
      float tv[8];
      if ((s0 >> 4) <= (r >> 4)) {
#pragma unroll
        for (int c = 0; c < 8; ++c) tv[c] = Tm[hp * (64 * PA_P) + r * PA_P + s0 + c] * bs[hp * 64 + s0 + c];
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) tv[c] = 0.0f;
      }
      uint4 hi, lo;
      tc::split8(tv, hi, lo);
      if (hp == 0 || gpair[1] != gpair[0]) {
        uint8_t* out = tp_ws + ((size_t)chunk * hv + j * G + gpair[hp]) * TP_BYTES;
        *reinterpret_cast<uint4*>(out + kmaj128(r, s0)) = hi;
        *reinterpret_cast<uint4*>(out + TP_TILE + kmaj128(r, s0)) = lo;
      }
      // the operand overwrites A: every thread must be past its last read of A (the
      // barrier above) -- and T lies outside the operand, so the reads here are safe
      const uint32_t boff = mnmaj(r, (hp * 64 + s0) >> 3, 64);
      *reinterpret_cast<uint4*>(pb_hi + boff) = hi;
      *reinterpret_cast<uint4*>(pb_lo + boff) = lo;
    }
    tc::fence_proxy_async();
    tc::tc_fence_before();
    __syncthreads();
    // P pair: D[128 x 128] = [Mq_a; Mq_b] (128 x 64) x [T_a | T_b] (64 x 128); the diagonal
    // blocks are P_a = Mq_a T_a (rows 0..63, cols 0..63) and P_b (rows 64..127, cols 64..127)
    if (tid == 0) {
      tc::tc_fence_after();
      constexpr uint32_t idesc = tc::idesc_bf16(128, 128, 0, 1);
      const uint64_t da[2] = {tc::sdesc(tc::smem_u32(pa_hi), LBO128, 128), tc::sdesc(tc::smem_u32(pa_lo), LBO128, 128)};
      const uint64_t db[2] = {tc::sdesc(tc::smem_u32(pb_hi), 128, 1024), tc::sdesc(tc::smem_u32(pb_lo), 128, 1024)};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int term = 0; term < 3; ++term)
          tc::umma_bf16(tbase + 128, da[term == 2] + (uint64_t)((ks * 2 * LBO128) >> 4),
                        db[term == 1] + (uint64_t)((ks * 256) >> 4), idesc, (ks | term) != 0);
      tc::umma_commit(tc::smem_u32(&mbar));
    }
    // warp-uniform, so that the warp-collective TMEM loads below run on every lane or none
    const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&mbar), mma_phase));
    mma_phase ^= 1;
    if (!ok) atomicExch(&g_gdn_status, -7);
    tc::tc_fence_after();
    if (warp < 4 && ok) {  // lane = hp * 64 + t: P row t of head hp, columns hp * 64 ..
      const int hp = tid >> 6, t = tid & 63;
      const uint32_t ta = tbase + 128 + ((uint32_t)(warp * 32) << 16) + hp * 64;
      uint32_t r0[32], r1[32];
      tc::tmem_ld32(ta, r0);
      tc::tmem_ld32(ta + 32, r1);
      tc::tmem_wait_ld();
      if (hp == 0 || gpair[1] != gpair[0]) {
        uint8_t* out = tp_ws + ((size_t)chunk * hv + j * G + gpair[hp]) * TP_BYTES;
#pragma unroll
        for (int s0 = 0; s0 < 64; s0 += 8) {
          float pv[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) pv[c] = __uint_as_float(s0 < 32 ? r0[s0 + c] : r1[s0 - 32 + c]);
          uint4 hi, lo;
          tc::split8(pv, hi, lo);
          *reinterpret_cast<uint4*>(out + kmaj128(64 + t, s0)) = hi;
          *reinterpret_cast<uint4*>(out + TP_TILE + kmaj128(64 + t, s0)) = lo;
        }
      }
    }
    tc::tc_fence_before();
    __syncthreads();
    // the next pair's raw v rows: the T matrices and the solve scratch are free again
    if (tid == 0 && ga + 2 < G && !s_abort) issue_v(ga + 2);
  }
  if (tid == 0) {
    tc::bulk_wait_all();  // the [K;Q] tile's bulk store has completed
    // after a timeout, let raw copies still in flight land (bounded): every arming of mbar_ld
    // but possibly the last was waited on, and the last completes the phase of parity ld_phase
    if (s_abort && ld_issued > ld_waited) (void)tc::mbar_wait(tc::smem_u32(&mbar_ld), ld_phase);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 256);
}

// ======================================================================================
// Phase B
// ======================================================================================
struct PBStage {  // byte offsets inside one input stage
  static constexpr uint32_t KQ = 0;
  static constexpr uint32_t TP = KQ_BYTES;
  static constexpr uint32_t GB = KQ_BYTES + TP_BYTES;
  static constexpr uint32_t VS = GB + GB_FLOATS * 4;  // v slice; later the R / U-tilde tile
  static constexpr uint32_t BYTES = VS + VS_SLICE;
};
constexpr uint32_t PB_S_TILE = 128 * TC_NV * 2;  // S^T operand (K = 128, N = nv), one of hi/lo
constexpr uint32_t PB_R_TILE = 64 * TC_NV * 2;   // R / U-tilde operand (K = 64, N = nv): 4 KB
constexpr size_t PB_TC_SMEM = 2 * (size_t)PB_S_TILE + 2 * (size_t)PBStage::BYTES;
static_assert(2 * PB_R_TILE == VS_SLICE, "the R / U-tilde tile reuses the v slot");

// Output modes of phase B: y before the output norm to the workspace (a separate epilogue
// follows), or the gated RMS norm fused in, with a bf16 or an fp32 y.
enum { PB_Y_RAW = 0, PB_Y_BF16 = 1, PB_Y_F32 = 2 };

// One CTA per (sequence, value head, 32-row state slice).  Warps 0..7 ("workers") serve TMEM
// lane quarter w % 4 and columns 16 (w / 4) .. 16 (w / 4) + 15 of the slice; warp 8 issues the
// bulk copies of the next chunk.  Each product a b is taken as a_hi [b_hi | b_lo] (one MMA of
// width 2 nv: the lo tile follows the hi tile at the operand's N stride) plus a_lo b_hi; the
// epilogue adds the two column halves.  (These small-N MMAs are bound by reading the A tile
// from shared memory, so two MMAs per k-step beat three of width nv.)  One barrier per chunk,
// at its start, orders the S tile, the stage reuse and the abort decision; a named barrier
// over the warps that own TMEM lanes 0..63 (warps 0, 1, 4, 5) hands R and U-tilde to the MMA
// thread between rounds.
//
// Fused output norm (YM != PB_Y_RAW; clusters of the four slices of a value head; 12 warps):
// warps 10 and 11 own TMEM lanes 64..127, i.e. the 64 tokens' y rows, and take the whole y
// path, so the workers only carry the state chain.  The norm of y_t over the head's 128
// components ("Qwen3.8-Flash-Next" technical report, Fig. 2: RMS norm of each head's output,
// gated by SiLU(z)) needs the sums of squares of all four slices: each norm thread stores its
// token's sum into the three other CTAs of the cluster as one 32-bit word whose two low bits
// carry a chunk tag (the value is the flag: no fence or barrier between CTAs), then waits for
// the peers' words and normalises its y row.  The norm warps stay out of the workers' chunk
// barriers: they arrive on per-parity mbarriers once they have read a chunk's gates and once
// they are done with its TMEM rows; the accumulators of rounds 1 and 2 are double-buffered by
// chunk parity, so thread 0 waits for the rows of chunk c - 2 only, and the producer reloads a
// stage only after the norm warps read its gates.  The exchange never holds up the state chain.  Every slice sums the same four tag-stripped words in rank order,
// so all four use the same norm.  Warp 9 idles.
template <int YM>
__global__ void __launch_bounds__(YM == PB_Y_RAW ? 288 : 384, 1)
    k_chunkscan_tc(Dims d, const int* __restrict__ cu, const int* __restrict__ seq_chunk0,
                   const int* __restrict__ order, const uint8_t* __restrict__ kq_ws, const uint8_t* __restrict__ tp_ws,
                   const float* __restrict__ gb_ws, const float* __restrict__ vs_ws,
                   const float* init_state, float* __restrict__ y_raw,
                   float* final_state,
                   const uint16_t* __restrict__ z, const float* __restrict__ norm_w, void* __restrict__ y) {
  constexpr int NV = TC_NV, NH = NV / 2;
  constexpr bool FUSED = YM != PB_Y_RAW;
  // blockIdx.x = (position * h_v + h) * 4 + slice: the four slices of a head are consecutive (one
  // cluster), and the sequences come in the tile map's order, longest first
  const int hq = d.h_qk, hv = d.h_v, G = hv / hq;
  const int sl = blockIdx.x % (D / NV), h = (blockIdx.x / (D / NV)) % hv, qpos = blockIdx.x / (D / NV) / hv;
  const int n = order ? order[qpos] : qpos, i0 = sl * NV, j = h / G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, cb = ((warp >> 2) & 1) * NH;
  const bool worker = warp < 8, producer = warp == 8;
  const bool normw = FUSED && warp >= 10;  // y rows of tokens 32 (warp - 10) + lane
  const bool rwarp = worker && quarter < 2;  // token rows 0..63: R and U-tilde
  const int row = quarter * 32 + lane;  // TMEM lane: accumulator row
  const int ts = cu ? cu[n] : 0, te = cu ? cu[n + 1] : d.total_tokens;
  const int nchunks = te > ts ? (te - ts + CH - 1) / CH : 0;
  const int gc0 = seq_chunk0 ? seq_chunk0[n] : 0;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* s_hi = sm;
  uint8_t* s_lo = sm + PB_S_TILE;
  uint8_t* stage[2] = {sm + 2 * PB_S_TILE, sm + 2 * PB_S_TILE + PBStage::BYTES};
  __shared__ uint64_t mbar_ld[2];
  // MMA completions: rounds 1 and 2 by chunk parity (their accumulators are double-buffered,
  // so the norm warps may read chunk c's rows while chunk c + 1 runs), round 3 once per chunk
  __shared__ uint64_t mbar_r1[2], mbar_r2[2], mbar_r3;
  __shared__ uint32_t tslot;
  __shared__ int s_abort;
  // fused norm, by chunk parity (64 arrivals each): the norm warps have read a chunk's gates
  // (the stage may be reloaded) and its TMEM rows (the accumulators may be reused)
  __shared__ uint64_t gates_read[2], norm_done[2];
  // fused norm: tagged sums of squares from the three other slices, [chunk parity][peer][token]
  __shared__ uint32_t red[FUSED ? 2 * 3 * 64 : 1];
  __shared__ __align__(16) float nw_s[FUSED ? NV : 4];  // fused norm: this slice's norm_w
  const int rank = FUSED ? (int)tc::cluster_ctarank() : 0;

  if (FUSED && tc::cluster_nctarank() != D / NV) {  // launched without its clusters: no exchange
    if (tid == 0) atomicExch(&g_gdn_status, -6);
    return;
  }
  // keep: a worker's state S[i0 + cb + i][row] (row = key component) in keep[0..15]; a norm
  // thread's pending y row in keep[0..31] (one register array serves both roles)
  float keep[NV];
  float* S = keep;
  const size_t sbase = (((size_t)n * hv + h) * D + i0) * D;
#pragma unroll
  for (int i = 0; i < NH; ++i) S[i] = (init_state && worker) ? init_state[sbase + (size_t)(cb + i) * D + row] : 0.0f;

  if (tid == 0) {
    s_abort = 0;
    tc::mbar_init(tc::smem_u32(&mbar_ld[0]), 1);
    tc::mbar_init(tc::smem_u32(&mbar_ld[1]), 1);
    for (int p2 = 0; p2 < 2; ++p2) {
      tc::mbar_init(tc::smem_u32(&mbar_r1[p2]), 1);
      tc::mbar_init(tc::smem_u32(&mbar_r2[p2]), 1);
      tc::mbar_init(tc::smem_u32(&gates_read[p2]), 64);
      tc::mbar_init(tc::smem_u32(&norm_done[p2]), 64);
    }
    tc::mbar_init(tc::smem_u32(&mbar_r3), 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(&tslot), 512);  // by chunk parity p: D_a 256 p + 0..63, D_cd 256 p + 64..127; D_e 128..191
    tc::tmem_relinquish();
  }
  // named barrier over a subset of the warps (id 1: the R / U-tilde writers, id 2: all but
  // the norm warps)
  auto named_bar_sync = [](int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
  };
  // the chunk barrier over every warp but the norm warps, returning the OR of `v` over them
  auto loop_sync_or = [&](bool v) -> bool {
    if (!FUSED) return __syncthreads_or(v) != 0;
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 2, 320, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
  };
  // A bounded wait that records a timeout.  Once any thread has recorded one, a later wait of
  // the CTA that does not complete at its first try returns at once (its barrier may never
  // complete), and the MMA thread issues no round after a failed wait, so the CTA reaches its
  // next chunk barrier, and leaves, within one limit.  The flag is read only off the fast path.
  auto aborted_now = [&]() { return *static_cast<volatile int*>(&s_abort) != 0; };
  auto wait_ok = [&](uint64_t& bar, uint32_t parity) -> bool {
    if (tc::mbar_try_wait(tc::smem_u32(&bar), parity)) return true;
    if (aborted_now()) return false;
    if (tc::mbar_wait(tc::smem_u32(&bar), parity)) return true;
    s_abort = 1;
    atomicExch(&g_gdn_status, -7);
    return false;
  };
  // (producer warp, lane 0) copies of chunk c into stage st
  auto issue_load = [&](int c, int st) {
    const size_t gc = (size_t)gc0 + c;
    const uint32_t bar = tc::smem_u32(&mbar_ld[st]);
    const uint32_t dst = tc::smem_u32(stage[st]);
    tc::mbar_arrive_expect_tx(bar, PBStage::BYTES);
    tc::bulk_g2s(dst + PBStage::KQ, kq_ws + (gc * hq + j) * KQ_BYTES, KQ_BYTES, bar);
    tc::bulk_g2s(dst + PBStage::TP, tp_ws + (gc * hv + h) * TP_BYTES, TP_BYTES, bar);
    tc::bulk_g2s(dst + PBStage::GB, gb_ws + (gc * hv + h) * GB_FLOATS, GB_FLOATS * 4, bar);
    tc::bulk_g2s(dst + PBStage::VS, vs_ws + (gc * hv + h) * (VS_BYTES / 4) + (size_t)sl * (VS_SLICE / 4), VS_SLICE,
                 bar);
  };
  // S^T operand: thread writes its row (K index = row) for its 16 columns, MN-major
  auto write_s_tile = [&]() {
#pragma unroll
    for (int q8 = 0; q8 < 2; ++q8) {
      uint4 hi, lo;
      tc::split8(S + q8 * 8, hi, lo);
      const uint32_t off = mnmaj(row, (cb >> 3) + q8, 128);
      *reinterpret_cast<uint4*>(s_hi + off) = hi;
      *reinterpret_cast<uint4*>(s_lo + off) = lo;
    }
  };
  if (worker) write_s_tile();
  if (FUSED) {
    for (int i = tid; i < 2 * 3 * 64; i += blockDim.x) red[i] = 3u;  // tag 3: no chunk yet
    if (tid < NV / 4) reinterpret_cast<float4*>(nw_s)[tid] = __ldg(reinterpret_cast<const float4*>(norm_w + i0) + tid);
  }
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();
  if (FUSED) tc::cluster_sync();  // peers started; their exchange words are initialised
  tc::tc_fence_after();
  const uint32_t tbase = tslot;
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  // accumulators (2 nv columns each: [a_hi b_hi + a_lo b_hi | a_hi b_lo])
  // accumulators; rounds 1 and 2 add 256 columns for odd chunks
  const uint32_t T_A = tbase, T_CD = tbase + 2 * NV, T_E = tbase + 4 * NV;
  const uint32_t t_a = T_A + lane_off + cb, t_cd = T_CD + lane_off + cb, t_e = T_E + lane_off + cb;
  auto par_cols = [](int c) { return (uint32_t)(c & 1) * 256u; };
  // The setup above reads only the call's inputs (the initial state may be the previous call's
  // final state: that call completed before this call's phase A started, and so before this
  // grid was launched) and overlaps phase A's last CTAs; phase A's tiles and gates are read
  // only from here on.
  tc::grid_dep_wait();
  tc::grid_dep_launch_dependents();
  int last_load = -1;  // (producer lane) the last chunk whose stage copies were issued
  if (producer && lane == 0 && nchunks > 0) {
    issue_load(0, 0);
    last_load = 0;
  }
  constexpr uint32_t idesc_kn2 = tc::idesc_bf16(128, 2 * NV, 0, 1);  // A K-major, B MN-major, N = 2 nv
  constexpr uint32_t idesc_kn = tc::idesc_bf16(128, NV, 0, 1);
  constexpr uint32_t idesc_mn2 = tc::idesc_bf16(128, 2 * NV, 1, 1);  // A and B MN-major
  constexpr uint32_t idesc_mn = tc::idesc_bf16(128, NV, 1, 1);
  const uint64_t d_s[2] = {tc::sdesc(tc::smem_u32(s_hi), 128, 16 * 128), tc::sdesc(tc::smem_u32(s_lo), 128, 16 * 128)};

  uint32_t ph_ld[2] = {0, 0};
  // phase parity of chunk c's completion on a barrier that completes once per chunk (round 3) or
  // once every two chunks (the per-parity barriers)
  auto ph1 = [](int c) { return (uint32_t)c & 1u; };
  auto ph2 = [](int c) { return (uint32_t)(c >> 1) & 1u; };
  bool aborted = false;
  // fused norm, norm threads: the previous chunk's y row (in keep, token y_tok, or -1)
  float* yv = keep;
  float own = 0.0f;
  int y_tok = -1;
  uint4 zcur[NV / 8];  // fused norm: the z row of this thread's token in the current chunk
  auto untag = [](uint32_t w) { return __uint_as_float(w & ~3u); };
  const uint32_t t_norm = tbase + ((uint32_t)(64 + 32 * (warp & 1)) << 16);  // norm warps: lanes 64.. / 96..
  // normalise and store the y row held from chunk cy (bounded wait for the peers' words)
  auto finish = [&](int cy) -> bool {
    const int t = row & 63, buf = cy & 1;
    const uint32_t tag = (uint32_t)(cy >> 1) & 3u;
    const uint32_t a0 = tc::smem_u32(&red[(buf * 3) * 64 + t]);
    uint32_t w[3];
    uint64_t t_start = 0;
    for (;;) {
#pragma unroll
      for (int p = 0; p < 3; ++p) w[p] = tc::ld_volatile_shared(a0 + p * 64 * 4);
      if ((w[0] & 3u) == tag && (w[1] & 3u) == tag && (w[2] & 3u) == tag) break;
      __nanosleep(64);
      uint64_t now;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
      if (t_start == 0) t_start = now;
      else if (now - t_start > g_gdn_wait_ns) return false;
    }
    float tot = 0.0f;  // the same words in the same order in every slice: identical norms
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
      tot += rr == rank ? own : untag(rr < rank ? w[rr < 3 ? rr : 2] : w[rr > 0 ? rr - 1 : 0]);
    if (y_tok >= 0) {
      const float inv = rsqrtf(tot * (1.0f / D) + d.rms_eps);
      const float4* nw4 = reinterpret_cast<const float4*>(nw_s);
      const size_t base = ((size_t)y_tok * hv + h) * D + i0;
#pragma unroll
      for (int g8 = 0; g8 < NV / 8; ++g8) {  // 8 columns at a time
        const uint4 zq = zcur[g8];
        const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
        const float4 wa = nw4[2 * g8], wb = nw4[2 * g8 + 1];
        float o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float zv = bf2f(u & 1 ? zw[u >> 1] >> 16 : zw[u >> 1] & 0xffffu);
          o[u] = yv[g8 * 8 + u] * inv * comp(u < 4 ? wa : wb, u & 3) * silu_fast(zv);
        }
        if (YM == PB_Y_BF16) {
          uint32_t pw[4];
#pragma unroll
          for (int u = 0; u < 8; u += 2) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(o[u], o[u + 1]);
            pw[u >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + base)[g8] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        } else {
          float4* yp = reinterpret_cast<float4*>(static_cast<float*>(y) + base) + 2 * g8;
          yp[0] = make_float4(o[0], o[1], o[2], o[3]);
          yp[1] = make_float4(o[4], o[5], o[6], o[7]);
        }
      }
    }
    return true;
  };
  // ---- fused norm: the y rows, one chunk behind nothing but the two MMA rounds they read ----
  if (normw) {
    const int t = row & 63;
    for (int c = 0; c < nchunks; ++c) {
      const int st = c & 1;
      const int t0 = ts + c * CH, L = min(CH, te - t0);
      if (t < L) {  // this token's z row, read now so that it has landed when the row is finished
        const uint4* zp = reinterpret_cast<const uint4*>(z + ((size_t)(t0 + t) * hv + h) * D + i0);
#pragma unroll
        for (int g8 = 0; g8 < NV / 8; ++g8) zcur[g8] = __ldg(zp + g8);
      }
      const float* gsm = reinterpret_cast<const float*>(stage[st] + PBStage::GB);
      // warp-uniform, so that the warp-collective TMEM loads run on every lane or none
      bool ok = __all_sync(0xffffffffu, wait_ok(mbar_ld[st], ph_ld[st]));
      ph_ld[st] ^= 1;
      const float eg = (ok && t < L) ? __expf(gsm[t]) : 0.0f;
      tc::mbar_arrive(tc::smem_u32(&gates_read[st]));  // the stage may be reloaded for chunk c + 2
      const uint32_t tn_c = t_norm + par_cols(c);
      float qs[NV];  // e^{gamma_t} (Q S^T)[t][:], all 32 columns of the slice, 16 at a time
      ok = __all_sync(0xffffffffu, ok && wait_ok(mbar_r1[st], ph2(c)));
      tc::tc_fence_after();
      if (ok) {
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
          uint32_t r[16], r2[16];
          tc::tmem_ld16(tn_c + 16 * h16, r);
          tc::tmem_ld16(tn_c + NV + 16 * h16, r2);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) qs[16 * h16 + i] = eg * (__uint_as_float(r[i]) + __uint_as_float(r2[i]));
        }
      }
      ok = __all_sync(0xffffffffu, ok && wait_ok(mbar_r2[st], ph2(c)));
      tc::tc_fence_after();
      if (ok) {  // Y = e^gamma Q S^T + (M o QK^T) U, and this slice's sum of squares to the peers
        float p = 0.0f;
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
          uint32_t r[16], r2[16];
          tc::tmem_ld16(tn_c + 2 * NV + 16 * h16, r);
          tc::tmem_ld16(tn_c + 3 * NV + 16 * h16, r2);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int k = 16 * h16 + i;
            yv[k] = t < L ? qs[k] + (__uint_as_float(r[i]) + __uint_as_float(r2[i])) : 0.0f;
            p = fmaf(yv[k], yv[k], p);
          }
        }
        y_tok = t < L ? t0 + t : -1;
        const int buf = c & 1;
        const uint32_t word = (__float_as_uint(p) & ~3u) | ((uint32_t)(c >> 1) & 3u);
        own = untag(word);
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          if (rr == rank) continue;
          const int slot = rank < rr ? rank : rank - 1;  // this slice's slot in peer rr
          tc::st_cluster_u32(tc::mapa(tc::smem_u32(&red[(buf * 3 + slot) * 64 + t]), (uint32_t)rr), word);
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(tc::smem_u32(&norm_done[st]));  // this chunk's TMEM rows are read
      // warp-uniform decisions: every lane of a norm warp leaves at the same chunk
      if (!__all_sync(0xffffffffu, ok && finish(c))) { s_abort = 1; atomicExch(&g_gdn_status, -7); break; }
      if (__any_sync(0xffffffffu, aborted_now())) break;
    }
  }
  for (int c = 0; c < nchunks && !aborted && !normw; ++c) {
    const int st = c & 1;
    const int t0 = ts + c * CH, L = min(CH, te - t0);
    uint8_t* sg = stage[st];
    uint8_t* r_hi = sg + PBStage::VS;
    uint8_t* r_lo = r_hi + PB_R_TILE;
    const uint32_t kq0 = tc::smem_u32(sg + PBStage::KQ), tp0 = tc::smem_u32(sg + PBStage::TP);
    if (worker) (void)wait_ok(mbar_ld[st], ph_ld[st]);
    ph_ld[st] ^= 1;
    const float* gsm = reinterpret_cast<const float*>(sg + PBStage::GB);
    const float gL = gsm[L - 1];
    const int t = row & 63;
    float vr[NH];  // R threads: v of token row t, read before the slot is reused
    if (rwarp) {
      const float4* vp = reinterpret_cast<const float4*>(sg + PBStage::VS) + (t * NV + cb) / 4;
#pragma unroll
      for (int q4 = 0; q4 < NH / 4; ++q4) {
        const float4 x = vp[q4];
        vr[q4 * 4 + 0] = x.x; vr[q4 * 4 + 1] = x.y; vr[q4 * 4 + 2] = x.z; vr[q4 * 4 + 3] = x.w;
      }
    }
    const float eg = t < L ? __expf(gsm[t]) : 0.0f;
    // the norm warps are done with the previous chunk's TMEM rows and stage before this
    // chunk's first round overwrites the one and the producer reloads the other
    // the norm warps are done with chunk c - 2's accumulator rows, which this chunk's rounds 1
    // and 2 overwrite
    if (FUSED && tid == 0 && c > 1) (void)wait_ok(norm_done[st], ph2(c - 2));
    // the chunk barrier, reducing the abort flag: a timeout recorded by any thread before it
    // arrived ends the loop for every thread at the same chunk
    if (loop_sync_or(aborted_now())) { aborted = true; break; }
    // ---- round 1: [K S^T ; Q S^T] = [K;Q] (128 x 128) x S^T (K = 128, N = nv) -------------
    if (tid == 0) {
      tc::tc_fence_after();
      const uint64_t da[2] = {tc::sdesc(kq0, LBO128, 128), tc::sdesc(kq0 + KQ_TILE, LBO128, 128)};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ao = (uint64_t)((ks * 2 * LBO128) >> 4), bo = (uint64_t)((ks * 256) >> 4);
        tc::umma_bf16(T_A + par_cols(c), da[0] + ao, d_s[0] + bo, idesc_kn2, ks != 0);  // a_hi [s_hi | s_lo]
        tc::umma_bf16(T_A + par_cols(c), da[1] + ao, d_s[0] + bo, idesc_kn, 1);         // a_lo s_hi
      }
      tc::umma_commit(tc::smem_u32(&mbar_r1[st]));
    }
    // the stage last read by chunk c - 1 (and, fused, its gates by the norm warps)
    if (producer && lane == 0 && c + 1 < nchunks && !aborted_now() &&
        (!FUSED || c == 0 || wait_ok(gates_read[st ^ 1], ph2(c - 1)))) {
      issue_load(c + 1, st ^ 1);
      last_load = c + 1;
    }
    const bool ok1 = wait_ok(mbar_r1[st], ph2(c));
    tc::tc_fence_after();
    float qs[NH];  // y rows (separate-epilogue mode): e^{gamma_t} (Q S^T)[t][:]
    if (rwarp || (!FUSED && worker)) {
      uint32_t r[16], r2[16];
      tc::tmem_ld16(t_a + par_cols(c), r);
      tc::tmem_ld16(t_a + par_cols(c) + NV, r2);
      tc::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) + __uint_as_float(r2[i]));
      if (quarter < 2) {  // R[t][i] = v[t][i] - e^{gamma_t} (K S^T)[t][i]  (beta is in the [T;P] tile)
        float rr[NH];
#pragma unroll
        for (int i = 0; i < NH; ++i) rr[i] = t < L ? fmaf(-eg, __uint_as_float(r[i]), vr[i]) : 0.0f;
#pragma unroll
        for (int q8 = 0; q8 < 2; ++q8) {
          uint4 hi, lo;
          tc::split8(rr + q8 * 8, hi, lo);
          const uint32_t off = mnmaj(t, (cb >> 3) + q8, 64);
          *reinterpret_cast<uint4*>(r_hi + off) = hi;
          *reinterpret_cast<uint4*>(r_lo + off) = lo;
        }
      } else {
#pragma unroll
        for (int i = 0; i < NH; ++i) qs[i] = eg * __uint_as_float(r[i]);
      }
    }
    tc::fence_proxy_async();
    tc::tc_fence_before();
    if (rwarp) named_bar_sync(1, 128);  // the R / U-tilde writers and the MMA thread
    // ---- round 2: [U ; (M o QK^T) U] = [T;P] (128 x 64) x R (K = 64, N = nv) ----------------
    if (tid == 0 && ok1) {
      tc::tc_fence_after();
      const uint64_t da[2] = {tc::sdesc(tp0, LBO128, 128), tc::sdesc(tp0 + TP_TILE, LBO128, 128)};
      const uint64_t db = tc::sdesc(tc::smem_u32(r_hi), 128, 8 * 128);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t ao = (uint64_t)((ks * 2 * LBO128) >> 4), bo = (uint64_t)((ks * 256) >> 4);
        tc::umma_bf16(T_CD + par_cols(c), da[0] + ao, db + bo, idesc_kn2, ks != 0);
        tc::umma_bf16(T_CD + par_cols(c), da[1] + ao, db + bo, idesc_kn, 1);
      }
      tc::umma_commit(tc::smem_u32(&mbar_r2[st]));
    }
    const bool ok2 = wait_ok(mbar_r2[st], ph2(c));
    tc::tc_fence_after();
    if (rwarp || (!FUSED && worker)) {
      uint32_t r[16], r2[16];
      tc::tmem_ld16(t_cd + par_cols(c), r);
      tc::tmem_ld16(t_cd + par_cols(c) + NV, r2);
      tc::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) + __uint_as_float(r2[i]));
      if (quarter < 2) {  // U-tilde[t][i] = e^{gamma_L - gamma_t} U[t][i]
        const float f = t < L ? __expf(gsm[64 + t]) : 0.0f;
        float uu[NH];
#pragma unroll
        for (int i = 0; i < NH; ++i) uu[i] = f * __uint_as_float(r[i]);
#pragma unroll
        for (int q8 = 0; q8 < 2; ++q8) {
          uint4 hi, lo;
          tc::split8(uu + q8 * 8, hi, lo);
          const uint32_t off = mnmaj(t, (cb >> 3) + q8, 64);
          *reinterpret_cast<uint4*>(r_hi + off) = hi;
          *reinterpret_cast<uint4*>(r_lo + off) = lo;
        }
      } else if (t < L) {  // Y = e^gamma Q S^T + (M o QK^T) U, before the output norm
        float4* yr = reinterpret_cast<float4*>(y_raw + ((size_t)(t0 + t) * hv + h) * D + i0 + cb);
#pragma unroll
        for (int q4 = 0; q4 < NH / 4; ++q4)
          yr[q4] = make_float4(qs[q4 * 4 + 0] + __uint_as_float(r[q4 * 4 + 0]),
                               qs[q4 * 4 + 1] + __uint_as_float(r[q4 * 4 + 1]),
                               qs[q4 * 4 + 2] + __uint_as_float(r[q4 * 4 + 2]),
                               qs[q4 * 4 + 3] + __uint_as_float(r[q4 * 4 + 3]));
      }
    }
    tc::fence_proxy_async();
    tc::tc_fence_before();
    if (rwarp) named_bar_sync(1, 128);  // the R / U-tilde writers and the MMA thread
    // ---- round 3: K^T U-tilde: A = MN-major view of the K rows (M = 128 key comps, K = 64 tokens)
    if (tid == 0 && ok2) {
      tc::tc_fence_after();
      const uint64_t da[2] = {tc::sdesc(kq0, 128, LBO128), tc::sdesc(kq0 + KQ_TILE, 128, LBO128)};
      const uint64_t db = tc::sdesc(tc::smem_u32(r_hi), 128, 8 * 128);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t o = (uint64_t)((ks * 256) >> 4);
        tc::umma_bf16(T_E, da[0] + o, db + o, idesc_mn2, ks != 0);
        tc::umma_bf16(T_E, da[1] + o, db + o, idesc_mn, 1);
      }
      tc::umma_commit(tc::smem_u32(&mbar_r3));
    }
    (void)wait_ok(mbar_r3, ph1(c));
    tc::tc_fence_after();
    if (worker) {
      uint32_t r[16], r2[16];
      tc::tmem_ld16(t_e, r);
      tc::tmem_ld16(t_e + NV, r2);
      tc::tmem_wait_ld();
      const float eL = __expf(gL);
#pragma unroll
      for (int i = 0; i < NH; ++i) S[i] = fmaf(eL, S[i], __uint_as_float(r[i]) + __uint_as_float(r2[i]));
      write_s_tile();
    }
    tc::fence_proxy_async();  // the next chunk's start barrier publishes the S tile
    tc::tc_fence_before();
  }
  if (!aborted && worker) {
#pragma unroll
    for (int i = 0; i < NH; ++i) final_state[sbase + (size_t)(cb + i) * D + row] = S[i];
  }
  // after a timeout, let the stage copies still in flight land (bounded) before the shared
  // memory they write is released: the last issued one completes its barrier's phase
  // (last_load >> 1) & 1, and every earlier one completed before it was waited on or before
  // the next copy into its stage was issued
  if (aborted_now() && producer && lane == 0 && last_load >= 0)
    (void)tc::mbar_wait(tc::smem_u32(&mbar_ld[last_load & 1]), (uint32_t)(last_load >> 1) & 1u);
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 512);
  if (FUSED) tc::cluster_sync();  // no CTA leaves while a peer may still write to it
}

}  // namespace gdn
