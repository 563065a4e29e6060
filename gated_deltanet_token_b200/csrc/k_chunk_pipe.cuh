// k_chunk_pipe.cuh -- phase B of the bf16 path with a software-pipelined chain (tcgen05).
//
// Same result as k_chunkscan_tc (field guide §02, steps 1-6, regrouped by chunks), with the
// sequential work per chunk cut to two MMA rounds.  The first product of chunk c + 1 splits as
//   [K;Q]_{c+1} S_{c+1}^T = e^{gamma_L} [K;Q]_{c+1} S_c^T + X_{c+1} U~_c,
//   X_{c+1} = [K;Q]_{c+1} K_c^T (phase A),  U~_c = diag(e^{gamma_L - gamma}) T R,
// since S_{c+1}^T = e^{gamma_L} S_c^T + K_c^T U~_c.  The state part ("early product") runs a
// chunk ahead, off the chain, into a second accumulator; the chain per chunk is
//   X U~ (K = 64) -> R -> [T;P] R (K = 64) -> U~,
// and the state update K^T U~ with its S-tile write runs beside it on other warps.
//
// Warps (12 with the fused output norm, 10 without):
//   0, 1, 4, 5  the chain: TMEM lanes 0..63 (token rows), R and U~, columns 16 (w / 4) ..
//   2, 3, 6, 7  state rows 64..127 (key components), 16 columns each; without the fused norm
//               also the y rows (TMEM lanes 64..127)
//   8, 9        state rows 0..63, all 32 columns; warp 8 lane 0 issues the bulk copies
//   10, 11      the fused output norm (as in k_chunkscan_tc)
// TMEM: first product (early part) 0..63, first product (X U~ part) 64..127, [T;P] R
// 128..191, K^T U~ 192..255, each two nv-column halves (a_hi [b_hi | b_lo] + a_lo b_hi).
#pragma once
#include "k_chunk_tc.cuh"

namespace gdn {

constexpr uint32_t PP_OFF_S = 0;                            // S^T tile hi | lo
constexpr uint32_t PP_OFF_KQ = 2 * PB_S_TILE;               // [K;Q] tiles by chunk parity
constexpr uint32_t PP_OFF_TP = PP_OFF_KQ + 2 * KQ_BYTES;    // [T;P] of the current chunk
constexpr uint32_t PP_OFF_X = PP_OFF_TP + TP_BYTES;         // X of the next chunk
constexpr uint32_t PP_OFF_R = PP_OFF_X + XT_BYTES;          // R hi | lo
constexpr uint32_t PP_OFF_U = PP_OFF_R + 2 * PB_R_TILE;     // U~ hi | lo
constexpr uint32_t PP_OFF_GB = PP_OFF_U + 2 * PB_R_TILE;    // gamma, beta by chunk parity
constexpr size_t PP_SMEM = PP_OFF_GB + 2 * GB_FLOATS * 4;
static_assert(PP_SMEM <= 225 * 1024, "pipelined phase B shared memory");

template <int YM>
__global__ void __launch_bounds__(YM == PB_Y_RAW ? 320 : 384, 1)
    k_chunkscan_pipe(Dims d, const int* __restrict__ cu, const int* __restrict__ seq_chunk0,
                     const uint8_t* __restrict__ kq_ws, const uint8_t* __restrict__ tp_ws,
                     const uint8_t* __restrict__ xt_ws, const float* __restrict__ gb_ws,
                     const float* __restrict__ vs_ws, const float* init_state, float* __restrict__ y_raw,
                     float* final_state, const uint16_t* __restrict__ z, const float* __restrict__ norm_w,
                     void* __restrict__ y) {
  tc::grid_dep_wait();  // phase A's tiles and gates are complete
  tc::grid_dep_launch_dependents();
  constexpr int NV = TC_NV, NH = NV / 2;
  constexpr bool FUSED = YM != PB_Y_RAW;
  const int n = blockIdx.x, h = blockIdx.y, sl = blockIdx.z, i0 = sl * NV;
  const int hq = d.h_qk, hv = d.h_v, G = hv / hq, j = h / G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, cb = ((warp >> 2) & 1) * NH;
  const bool chain = warp < 8 && quarter < 2;
  const bool q23 = warp < 8 && quarter >= 2;
  const bool s01 = warp == 8 || warp == 9;
  const bool sown = q23 || s01;
  const bool producer = warp == 8;
  const bool normw = FUSED && warp >= 10;
  const bool ywarp = !FUSED && q23;
  const int row = quarter * 32 + lane;  // TMEM lane
  const int ts = cu ? cu[n] : 0, te = cu ? cu[n + 1] : d.total_tokens;
  const int nchunks = te > ts ? (te - ts + CH - 1) / CH : 0;
  const int gc0 = seq_chunk0 ? seq_chunk0[n] : 0;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* s_hi = sm + PP_OFF_S;
  uint8_t* s_lo = s_hi + PB_S_TILE;
  uint8_t* kqb[2] = {sm + PP_OFF_KQ, sm + PP_OFF_KQ + KQ_BYTES};
  uint8_t* tpb = sm + PP_OFF_TP;
  uint8_t* xb = sm + PP_OFF_X;
  uint8_t* r_hi = sm + PP_OFF_R;
  uint8_t* r_lo = r_hi + PB_R_TILE;
  uint8_t* u_hi = sm + PP_OFF_U;
  uint8_t* u_lo = u_hi + PB_R_TILE;
  float* gbb[2] = {reinterpret_cast<float*>(sm + PP_OFF_GB), reinterpret_cast<float*>(sm + PP_OFF_GB) + GB_FLOATS};
  __shared__ uint64_t mbar_gb[2], mbar_kq[2], mbar_tp, mbar_x;
  // MMA completions, once per chunk each: the chunk's first product; round 2; K^T U~
  __shared__ uint64_t mbar_first, mbar_r2, mbar_state;
  __shared__ uint64_t qread;      // fused norm: the norm warps have read the chunk's first product
  __shared__ uint64_t norm_done;  // the y-row threads have read the chunk's [T;P] R rows 64..127
  __shared__ uint32_t tslot;
  __shared__ int s_abort;
  __shared__ uint32_t red[FUSED ? 2 * 3 * 64 : 1];
  const int rank = FUSED ? (int)tc::cluster_ctarank() : 0;

  if (FUSED && tc::cluster_nctarank() != D / NV) {
    if (tid == 0) atomicExch(&g_gdn_status, -6);
    return;
  }
  // keep: a state owner's S[i0 + c0s + i][row] for i < ncol; a norm thread's pending y row
  float keep[NV];
  float* S = keep;
  const int ncol = s01 ? NV : NH, c0s = s01 ? 0 : cb;
  const size_t sbase = (((size_t)n * hv + h) * D + i0) * D;
#pragma unroll
  for (int i = 0; i < NV; ++i)
    S[i] = (sown && i < ncol && init_state) ? init_state[sbase + (size_t)(c0s + i) * D + row] : 0.0f;

  if (tid == 0) {
    s_abort = 0;
    for (int b2 = 0; b2 < 2; ++b2) {
      tc::mbar_init(tc::smem_u32(&mbar_gb[b2]), 1);
      tc::mbar_init(tc::smem_u32(&mbar_kq[b2]), 1);
    }
    tc::mbar_init(tc::smem_u32(&mbar_tp), 1);
    tc::mbar_init(tc::smem_u32(&mbar_x), 1);
    tc::mbar_init(tc::smem_u32(&mbar_first), 1);
    tc::mbar_init(tc::smem_u32(&mbar_r2), 1);
    tc::mbar_init(tc::smem_u32(&mbar_state), 1);
    tc::mbar_init(tc::smem_u32(&qread), 64);
    tc::mbar_init(tc::smem_u32(&norm_done), FUSED ? 64 : 128);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(&tslot), 256);
    tc::tmem_relinquish();
  }
  auto named_bar_sync = [](int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
  };
  auto loop_sync = [&]() { named_bar_sync(2, 320); };  // every warp but the norm warps
  auto wait = [&](uint64_t& bar, uint32_t parity) -> bool {
    const bool ok = tc::mbar_wait(tc::smem_u32(&bar), parity);
    if (!ok) {
      s_abort = 1;
      atomicExch(&g_gdn_status, -7);
    }
    return ok;
  };
  // (producer lane) bulk copies of chunk c
  auto issue_gb = [&](int c) {
    const uint32_t bar = tc::smem_u32(&mbar_gb[c & 1]);
    tc::mbar_arrive_expect_tx(bar, GB_FLOATS * 4);
    tc::bulk_g2s(tc::smem_u32(gbb[c & 1]), gb_ws + ((size_t)(gc0 + c) * hv + h) * GB_FLOATS, GB_FLOATS * 4, bar);
  };
  auto kq_src = [&](int c) { return kq_ws + ((size_t)(gc0 + c) * hq + j) * KQ_BYTES; };
  auto issue_kq = [&](int c) {
    const uint32_t bar = tc::smem_u32(&mbar_kq[c & 1]);
    tc::mbar_arrive_expect_tx(bar, KQ_BYTES);
    tc::bulk_g2s(tc::smem_u32(kqb[c & 1]), kq_src(c), KQ_BYTES, bar);
  };
  auto issue_tp = [&](int c) {
    const uint32_t bar = tc::smem_u32(&mbar_tp);
    tc::mbar_arrive_expect_tx(bar, TP_BYTES);
    tc::bulk_g2s(tc::smem_u32(tpb), tp_ws + ((size_t)(gc0 + c) * hv + h) * TP_BYTES, TP_BYTES, bar);
  };
  auto issue_x = [&](int c) {
    const uint32_t bar = tc::smem_u32(&mbar_x);
    tc::mbar_arrive_expect_tx(bar, XT_BYTES);
    tc::bulk_g2s(tc::smem_u32(xb), xt_ws + ((size_t)(gc0 + c) * hq + j) * XT_BYTES, XT_BYTES, bar);
  };
  // S^T operand: a state owner writes its row (K index = row) for its columns, MN-major
  auto write_s_tile = [&]() {
#pragma unroll
    for (int q8 = 0; q8 < NV / 8; ++q8) {
      if (q8 * 8 >= ncol) break;
      uint4 hi, lo;
      tc::split8(S + q8 * 8, hi, lo);
      const uint32_t off = mnmaj(row, (c0s >> 3) + q8, 128);
      *reinterpret_cast<uint4*>(s_hi + off) = hi;
      *reinterpret_cast<uint4*>(s_lo + off) = lo;
    }
  };
  // chain threads: v of token row t of chunk c (this slice's 16 columns), one chunk ahead
  const int t = row & 63;
  float vnext[NH];
  auto load_v = [&](int c) {
    const float4* vp = reinterpret_cast<const float4*>(vs_ws + ((size_t)(gc0 + c) * hv + h) * (VS_BYTES / 4) +
                                                       (size_t)sl * (VS_SLICE / 4) + t * NV + cb);
#pragma unroll
    for (int q4 = 0; q4 < NH / 4; ++q4) {
      const float4 x = __ldg(vp + q4);
      vnext[q4 * 4 + 0] = x.x; vnext[q4 * 4 + 1] = x.y; vnext[q4 * 4 + 2] = x.z; vnext[q4 * 4 + 3] = x.w;
    }
  };
  if (sown) write_s_tile();
  if (FUSED)
    for (int i = tid; i < 2 * 3 * 64; i += blockDim.x) red[i] = 3u;
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();
  if (FUSED) tc::cluster_sync();
  tc::tc_fence_after();
  const uint32_t tbase = tslot;
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  const uint32_t T_A1 = tbase, T_A2 = tbase + 2 * NV, T_CD = tbase + 4 * NV, T_E = tbase + 6 * NV;
  const uint32_t t_a1 = T_A1 + lane_off + cb, t_a2 = T_A2 + lane_off + cb, t_cd = T_CD + lane_off + cb;
  const uint32_t t_e = T_E + lane_off + c0s;
  constexpr uint32_t idesc_kn2 = tc::idesc_bf16(128, 2 * NV, 0, 1);  // A K-major, B MN-major, N = 2 nv
  constexpr uint32_t idesc_kn = tc::idesc_bf16(128, NV, 0, 1);
  constexpr uint32_t idesc_mn2 = tc::idesc_bf16(128, 2 * NV, 1, 1);  // A and B MN-major
  constexpr uint32_t idesc_mn = tc::idesc_bf16(128, NV, 1, 1);
  const uint64_t d_s = tc::sdesc(tc::smem_u32(s_hi), 128, 16 * 128);
  const uint64_t d_r = tc::sdesc(tc::smem_u32(r_hi), 128, 8 * 128);
  const uint64_t d_u = tc::sdesc(tc::smem_u32(u_hi), 128, 8 * 128);
  // [K;Q] (128 x 128) x S^T (K = 128, N = nv) into accumulator acc
  auto issue_kq_s = [&](const uint8_t* kq, uint32_t acc) {
    const uint32_t k0 = tc::smem_u32(kq);
    const uint64_t da[2] = {tc::sdesc(k0, LBO128, 128), tc::sdesc(k0 + KQ_TILE, LBO128, 128)};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint64_t ao = (uint64_t)((ks * 2 * LBO128) >> 4), bo = (uint64_t)((ks * 256) >> 4);
      tc::umma_bf16(acc, da[0] + ao, d_s + bo, idesc_kn2, ks != 0);
      tc::umma_bf16(acc, da[1] + ao, d_s + bo, idesc_kn, 1);
    }
  };
  // A (128 x 64, K-major tiles hi | lo at a0, a0 + TP_TILE) x B (K = 64, N = nv) into acc
  auto issue_k64 = [&](uint32_t a0, uint64_t db, uint32_t acc) {
    const uint64_t da[2] = {tc::sdesc(a0, LBO128, 128), tc::sdesc(a0 + TP_TILE, LBO128, 128)};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint64_t ao = (uint64_t)((ks * 2 * LBO128) >> 4), bo = (uint64_t)((ks * 256) >> 4);
      tc::umma_bf16(acc, da[0] + ao, db + bo, idesc_kn2, ks != 0);
      tc::umma_bf16(acc, da[1] + ao, db + bo, idesc_kn, 1);
    }
  };
  if (producer && lane == 0 && nchunks > 0) {
    issue_gb(0);
    issue_kq(0);
    issue_tp(0);
    if (nchunks > 1) {
      issue_gb(1);
      issue_kq(1);
      issue_x(1);
    }
    if (nchunks > 2) tc::prefetch_l2(kq_src(2), KQ_BYTES);
  }
  if (chain && nchunks > 0) load_v(0);
  if (tid == 0 && nchunks > 0 && wait(mbar_kq[0], 0)) {  // chunk 0's first product: round 1 on S_0
    tc::tc_fence_after();
    issue_kq_s(kqb[0], T_A1);
    tc::umma_commit(tc::smem_u32(&mbar_first));
  }

  bool aborted = false;
  float eLp = 1.0f;  // e^{gamma_L} of the previous chunk
  float* yv = keep;  // norm threads: the previous chunk's y row
  float own = 0.0f;
  int y_tok = -1;
  auto untag = [](uint32_t w) { return __uint_as_float(w & ~3u); };
  const uint32_t t_norm = tbase + ((uint32_t)(64 + 32 * (warp & 1)) << 16);
  // normalise and store the y row held from chunk cy (bounded wait for the peers' words)
  auto finish = [&](int cy) -> bool {
    const int tt = row & 63, buf = cy & 1;
    const uint32_t tag = (uint32_t)(cy >> 1) & 3u;
    const uint32_t a0 = tc::smem_u32(&red[(buf * 3) * 64 + tt]);
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
      else if (now - t_start > 2000000000ull) return false;
    }
    float tot = 0.0f;
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
      tot += rr == rank ? own : untag(rr < rank ? w[rr < 3 ? rr : 2] : w[rr > 0 ? rr - 1 : 0]);
    if (y_tok >= 0) {
      const float inv = rsqrtf(tot * (1.0f / D) + d.rms_eps);
      const float4* nw4 = reinterpret_cast<const float4*>(norm_w + i0);
      const size_t base = ((size_t)y_tok * hv + h) * D + i0;
      const uint4* zp = reinterpret_cast<const uint4*>(z + base);
#pragma unroll
      for (int g8 = 0; g8 < NV / 8; ++g8) {
        const uint4 zq = __ldg(zp + g8);
        const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
        const float4 wa = __ldg(nw4 + 2 * g8), wb = __ldg(nw4 + 2 * g8 + 1);
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

  // ---- fused norm warps: the y rows of each chunk --------------------------------------
  if (normw) {
    const int tt = row & 63;
    for (int c = 0; c < nchunks; ++c) {
      const int st = c & 1;
      const int t0 = ts + c * CH, L = min(CH, te - t0);
      const float* gsm = gbb[st];
      bool ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&mbar_gb[st]), (uint32_t)(c >> 1) & 1u));
      const float eg = (ok && tt < L) ? __expf(gsm[tt]) : 0.0f;
      const float eL = ok ? __expf(gsm[L - 1]) : 0.0f;
      float qs[NV];  // e^{gamma_t} (Q S_c^T)[t][:], all 32 columns of the slice
      ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(tc::smem_u32(&mbar_first), (uint32_t)c & 1u));
      tc::tc_fence_after();
      if (ok) {
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
          uint32_t r[16], r2[16];
          tc::tmem_ld16(t_norm + 16 * h16, r);
          tc::tmem_ld16(t_norm + NV + 16 * h16, r2);
          tc::tmem_wait_ld();
          float f[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(r[i]) + __uint_as_float(r2[i]);
          if (c > 0) {
            tc::tmem_ld16(t_norm + 2 * NV + 16 * h16, r);
            tc::tmem_ld16(t_norm + 3 * NV + 16 * h16, r2);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) f[i] = fmaf(eLp, f[i], __uint_as_float(r[i]) + __uint_as_float(r2[i]));
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) qs[16 * h16 + i] = eg * f[i];
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(tc::smem_u32(&qread));  // the early product of chunk c + 1 may overwrite these
      eLp = eL;
      ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(tc::smem_u32(&mbar_r2), (uint32_t)c & 1u));
      tc::tc_fence_after();
      if (ok) {  // Y = e^gamma Q S^T + (M o QK^T) U, and this slice's sum of squares to the peers
        float p = 0.0f;
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
          uint32_t r[16], r2[16];
          tc::tmem_ld16(t_norm + 4 * NV + 16 * h16, r);
          tc::tmem_ld16(t_norm + 5 * NV + 16 * h16, r2);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int k = 16 * h16 + i;
            yv[k] = tt < L ? qs[k] + (__uint_as_float(r[i]) + __uint_as_float(r2[i])) : 0.0f;
            p = fmaf(yv[k], yv[k], p);
          }
        }
        y_tok = tt < L ? t0 + tt : -1;
        const int buf = c & 1;
        const uint32_t word = (__float_as_uint(p) & ~3u) | ((uint32_t)(c >> 1) & 3u);
        own = untag(word);
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          if (rr == rank) continue;
          const int slot = rank < rr ? rank : rank - 1;
          tc::st_cluster_u32(tc::mapa(tc::smem_u32(&red[(buf * 3 + slot) * 64 + tt]), (uint32_t)rr), word);
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(tc::smem_u32(&norm_done));
      if (!ok || !finish(c)) { s_abort = 1; atomicExch(&g_gdn_status, -7); break; }
      if (s_abort) break;
    }
  }

  // ---- every other warp ------------------------------------------------------------------
  for (int c = 0; c < nchunks && !aborted && !normw; ++c) {
    const int st = c & 1;
    const int t0 = ts + c * CH, L = min(CH, te - t0);
    const float* gsm = gbb[st];
    bool ok = __all_sync(0xffffffffu, wait(mbar_gb[st], (uint32_t)(c >> 1) & 1u));
    const float gL = ok ? gsm[L - 1] : 0.0f;
    const float eg = (ok && t < L) ? __expf(gsm[t]) : 0.0f;
    const float bt = (ok && t < L) ? gsm[64 + t] : 0.0f;
    float vr[NH];
    if (chain) {
#pragma unroll
      for (int i = 0; i < NH; ++i) vr[i] = vnext[i];
      if (c + 1 < nchunks) load_v(c + 1);
    }
    // B: the chunk's first product (round 1 for chunk 0, else e^{gamma_L} early + X U~)
    ok = __all_sync(0xffffffffu, ok && wait(mbar_first, (uint32_t)c & 1u));
    tc::tc_fence_after();
    if (producer && lane == 0 && ok && c >= 1 && c + 1 < nchunks) issue_x(c + 1);  // X(c) is read
    float f[NH];
    float qs[NH];
    if ((chain || ywarp) && ok) {
      uint32_t r[16], r2[16];
      tc::tmem_ld16(t_a1, r);
      tc::tmem_ld16(t_a1 + NV, r2);
      tc::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < NH; ++i) f[i] = __uint_as_float(r[i]) + __uint_as_float(r2[i]);
      if (c > 0) {
        tc::tmem_ld16(t_a2, r);
        tc::tmem_ld16(t_a2 + NV, r2);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < NH; ++i) f[i] = fmaf(eLp, f[i], __uint_as_float(r[i]) + __uint_as_float(r2[i]));
      }
      if (chain) {  // R[t][i] = beta_t (v[t][i] - e^{gamma_t} (K S^T)[t][i])
        float rr[NH];
#pragma unroll
        for (int i = 0; i < NH; ++i) rr[i] = t < L ? bt * fmaf(-eg, f[i], vr[i]) : 0.0f;
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
        for (int i = 0; i < NH; ++i) qs[i] = eg * f[i];
      }
    }
    tc::fence_proxy_async();
    tc::tc_fence_before();
    if (chain) named_bar_sync(1, 128);  // R is written
    // C: round 2, [U ; (M o QK^T) U] = [T;P] (128 x 64) x R
    if (tid == 0 && ok) {
      tc::tc_fence_after();
      bool w = true;
      if (c > 0) w = wait(norm_done, (uint32_t)(c - 1) & 1u);  // chunk c-1's y rows are read
      w = w && wait(mbar_tp, (uint32_t)c & 1u);
      if (w) {
        issue_k64(tc::smem_u32(tpb), d_r, T_CD);
        tc::umma_commit(tc::smem_u32(&mbar_r2));
      }
    }
    // H(c-1): the previous chunk's state update, beside round 2
    if (sown && c > 0) {
      const bool okc = __all_sync(0xffffffffu, wait(mbar_state, (uint32_t)(c - 1) & 1u));
      tc::tc_fence_after();
      if (okc) {
#pragma unroll
        for (int h16 = 0; h16 < NV / 16; ++h16) {
          if (h16 * 16 >= ncol) break;
          uint32_t r[16], r2[16];
          tc::tmem_ld16(t_e + 16 * h16, r);
          tc::tmem_ld16(t_e + NV + 16 * h16, r2);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            S[16 * h16 + i] = fmaf(eLp, S[16 * h16 + i], __uint_as_float(r[i]) + __uint_as_float(r2[i]));
        }
        write_s_tile();
      }
      if (producer && lane == 0 && okc && c + 1 < nchunks) {  // K^T U~ of chunk c-1 has read its tile
        issue_kq(c + 1);
        if (c + 2 < nchunks) tc::prefetch_l2(kq_src(c + 2), KQ_BYTES);
      }
    }
    tc::fence_proxy_async();  // the chunk barrier publishes the S tile
    tc::tc_fence_before();
    // D: the S_c tile is written and the chunk's first product read by every warp here
    loop_sync();
    if (s_abort) { aborted = true; break; }
    if (producer && lane == 0 && c >= 1 && c + 1 < nchunks) {  // the gates of chunk c+1
      if (!FUSED || wait(norm_done, (uint32_t)(c - 1) & 1u)) issue_gb(c + 1);
    }
    // E: the early product of chunk c+1, [K;Q]_{c+1} S_c^T, off the chain
    if (tid == 0 && c + 1 < nchunks) {
      tc::tc_fence_after();
      bool w = !FUSED || wait(qread, (uint32_t)c & 1u);
      w = w && wait(mbar_kq[(c + 1) & 1], (uint32_t)((c + 1) >> 1) & 1u);
      if (w) issue_kq_s(kqb[(c + 1) & 1], T_A1);
    }
    // F: U~ (chain) and the y rows without the fused norm
    bool ok2 = false;
    if (chain || ywarp || producer) ok2 = __all_sync(0xffffffffu, wait(mbar_r2, (uint32_t)c & 1u));
    tc::tc_fence_after();
    if (producer && lane == 0 && ok2 && c + 1 < nchunks) issue_tp(c + 1);  // round 2 has read [T;P]
    if ((chain || ywarp) && ok2) {
      uint32_t r[16], r2[16];
      tc::tmem_ld16(t_cd, r);
      tc::tmem_ld16(t_cd + NV, r2);
      tc::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) + __uint_as_float(r2[i]));
      if (chain) {  // U~[t][i] = e^{gamma_L - gamma_t} U[t][i]
        const float ft = t < L ? __expf(gL - gsm[t]) : 0.0f;
        float uu[NH];
#pragma unroll
        for (int i = 0; i < NH; ++i) uu[i] = ft * __uint_as_float(r[i]);
#pragma unroll
        for (int q8 = 0; q8 < 2; ++q8) {
          uint4 hi, lo;
          tc::split8(uu + q8 * 8, hi, lo);
          const uint32_t off = mnmaj(t, (cb >> 3) + q8, 64);
          *reinterpret_cast<uint4*>(u_hi + off) = hi;
          *reinterpret_cast<uint4*>(u_lo + off) = lo;
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
    if (ywarp) {
      tc::tc_fence_before();
      tc::mbar_arrive(tc::smem_u32(&norm_done));  // round 2 of chunk c+1 may overwrite these rows
    }
    tc::fence_proxy_async();
    tc::tc_fence_before();
    if (chain) named_bar_sync(1, 128);  // U~ is written
    // G: the next chunk's first product X_{c+1} U~ (the chain), then K^T U~ (the state)
    if (tid == 0) {
      tc::tc_fence_after();
      if (c + 1 < nchunks && wait(mbar_x, (uint32_t)c & 1u)) {
        issue_k64(tc::smem_u32(xb), d_u, T_A2);
        tc::umma_commit(tc::smem_u32(&mbar_first));
      }
      const uint32_t k0 = tc::smem_u32(kqb[c & 1]);
      const uint64_t da[2] = {tc::sdesc(k0, 128, LBO128), tc::sdesc(k0 + KQ_TILE, 128, LBO128)};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t o = (uint64_t)((ks * 256) >> 4);
        tc::umma_bf16(T_E, da[0] + o, d_u + o, idesc_mn2, ks != 0);
        tc::umma_bf16(T_E, da[1] + o, d_u + o, idesc_mn, 1);
      }
      tc::umma_commit(tc::smem_u32(&mbar_state));
    }
    eLp = __expf(gL);
  }
  // the last chunk's state update
  if (!aborted && !normw && sown && nchunks > 0) {
    const bool okc = __all_sync(0xffffffffu, wait(mbar_state, (uint32_t)(nchunks - 1) & 1u));
    tc::tc_fence_after();
    if (okc) {
#pragma unroll
      for (int h16 = 0; h16 < NV / 16; ++h16) {
        if (h16 * 16 >= ncol) break;
        uint32_t r[16], r2[16];
        tc::tmem_ld16(t_e + 16 * h16, r);
        tc::tmem_ld16(t_e + NV + 16 * h16, r2);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          S[16 * h16 + i] = fmaf(eLp, S[16 * h16 + i], __uint_as_float(r[i]) + __uint_as_float(r2[i]));
      }
    } else {
      aborted = true;
    }
  }
  if (!aborted && sown) {
#pragma unroll
    for (int i = 0; i < NV; ++i)
      if (i < ncol) final_state[sbase + (size_t)(c0s + i) * D + row] = S[i];
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, 256);
  if (FUSED) tc::cluster_sync();
}

}  // namespace gdn
