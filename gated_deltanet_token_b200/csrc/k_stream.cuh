// k_stream.cuh -- the streaming kernels of the prefill: varlen tile map (K3), the
// conv + SiLU + L2-norm + gate prologue (K1) and the gated-RMSNorm epilogue (K5).
#pragma once
#include "gdn_common.cuh"

namespace gdn {

// ---- K3: varlen tile map -------------------------------------------------------------
// One block.  From cu_seqlens (device; NULL = one sequence of T_tot tokens) builds the
// chunk table (one entry per 64-token chunk, chunks aligned to sequence starts) and
// seq_chunk0[n] = index of sequence n's first chunk (seq_chunk0[N] = total chunks).
// Runs on the device, so the host never reads cu_seqlens.
// Also, when `order` is given, the order in which phase B takes the sequences: by chunk count,
// longest first (ties by index), so that the longest state chains start in the first wave of
// CTAs; beyond TILEMAP_ORDER_MAX sequences, index order.
constexpr int TILEMAP_ORDER_MAX = 1024;
__global__ void __launch_bounds__(1024) k_tilemap(const int* __restrict__ cu, int N, int T_tot,
                                                  int max_chunks, ChunkEntry* __restrict__ tab,
                                                  int* __restrict__ seq_chunk0, int* __restrict__ order) {
  __shared__ int s_nc[TILEMAP_ORDER_MAX];
  __shared__ int s_warp[32];
  __shared__ int s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < N; base += blockDim.x) {
    const int n = base + tid;
    int nc = 0;
    if (n < N) {
      const int a = cu ? cu[n] : 0, b = cu ? cu[n + 1] : T_tot;
      nc = b > a ? (b - a + CH - 1) / CH : 0;
    }
    int x = nc;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < nw) s_warp[lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    const int incl = x + (warp ? s_warp[warp - 1] : 0) + s_carry;
    if (n < N) seq_chunk0[n] = incl - nc;
    __syncthreads();
    if (tid == blockDim.x - 1) s_carry = incl;
    __syncthreads();
  }
  if (tid == 0) seq_chunk0[N] = s_carry;
  __syncthreads();
  if (order) {
    if (N <= TILEMAP_ORDER_MAX) {
      for (int n = tid; n < N; n += blockDim.x) s_nc[n] = seq_chunk0[n + 1] - seq_chunk0[n];
      __syncthreads();
      for (int n = tid; n < N; n += blockDim.x) {
        const int mine = s_nc[n];
        int rank = 0;
        for (int m = 0; m < N; ++m) {
          const int other = s_nc[m];
          rank += (other > mine) || (other == mine && m < n);
        }
        order[rank] = n;
      }
    } else {
      for (int n = tid; n < N; n += blockDim.x) order[n] = n;
    }
  }
  const int total = s_carry;
  for (int c = tid; c < max_chunks; c += blockDim.x) {
    ChunkEntry e{0, 0, 0, 0};
    if (c < total) {
      int lo = 0, hi = N - 1;  // largest n with seq_chunk0[n] <= c
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seq_chunk0[mid] <= c) lo = mid; else hi = mid - 1;
      }
      const int a = cu ? cu[lo] : 0, b = cu ? cu[lo + 1] : T_tot;
      e.seq = lo;
      e.t0 = a + (c - seq_chunk0[lo]) * CH;
      e.len = min(CH, b - e.t0);
      e.seq_start = a;
    }
    tab[c] = e;
  }
}

// ---- K1: prologue ----------------------------------------------------------------------
// Grid (chunk, head unit); head unit u < h_qk: q head u; < 2 h_qk: k head; else v head.
// Each warp takes 8 consecutive tokens of the chunk with its 3-token conv history, each
// lane 4 channels.  Per token: width-4 causal conv, SiLU ("Qwen3.8-Flash-Next" technical
// report, Fig. 2; field guide §02: width-4 depthwise causal conv); q and k are then
// L2-normalised (Fig. 2) -- q also scaled by q_scale.  Value-head units also compute the
// gates g (decay-gate note of the model notes) and beta = sigmoid(b) per token.
// Outputs are fp32 rows [T][heads][128]; g, beta are [T][h_v].
template <bool BF16>
__global__ void __launch_bounds__(256) k_prologue(Dims d, const ChunkEntry* __restrict__ tab,
                                                  const void* __restrict__ q, const void* __restrict__ k,
                                                  const void* __restrict__ v, const float* __restrict__ a,
                                                  const float* __restrict__ b,
                                                  const float* __restrict__ A_log,
                                                  const float* __restrict__ dt_bias,
                                                  const float* __restrict__ conv_w, float* __restrict__ qn,
                                                  float* __restrict__ kn, float* __restrict__ vc,
                                                  float* __restrict__ g_out, float* __restrict__ beta_out) {
  const ChunkEntry e = tab[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tb = warp * 8;
  if (e.len == 0 || tb >= e.len) return;
  const int u = blockIdx.y, hq = d.h_qk, hv = d.h_v;
  const void* src;
  float* dst;
  int nheads, head;
  size_t ch0;
  bool norm;
  float scale = 1.0f;
  if (u < hq) {
    src = q; dst = qn; nheads = hq; head = u; ch0 = (size_t)u * D; norm = true; scale = d.q_scale;
  } else if (u < 2 * hq) {
    src = k; dst = kn; nheads = hq; head = u - hq; ch0 = (size_t)(hq + head) * D; norm = true;
  } else {
    src = v; dst = vc; nheads = hv; head = u - 2 * hq; ch0 = (size_t)(2 * hq) * D + (size_t)head * D;
    norm = false;
  }
  const int c0 = lane * 4;
  float w[4][4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 t = *reinterpret_cast<const float4*>(conv_w + (ch0 + c0 + c) * 4);
    w[c][0] = t.x; w[c][1] = t.y; w[c][2] = t.z; w[c][3] = t.w;
  }
  // window: positions tb-3 .. tb+7 of the chunk
  float4 x[11];
#pragma unroll
  for (int p = 0; p < 11; ++p) {
    const int tc = tb - 3 + p;            // chunk-relative token
    const long tg = (long)e.t0 + tc;      // packed token
    const bool ok = tc < e.len && tg >= e.seq_start;
    x[p] = ok ? load4<BF16>(src, ((size_t)tg * nheads + head) * D + c0) : make_float4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (tb + i >= e.len) break;  // warp-uniform
    float r[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float acc = fmaf(w[c][3], comp(x[i + 3], c),
                             fmaf(w[c][2], comp(x[i + 2], c),
                                  fmaf(w[c][1], comp(x[i + 1], c), w[c][0] * comp(x[i], c))));
      r[c] = silu_f(acc);
    }
    if (norm) {
      const float ss = warp_sum(r[0] * r[0] + r[1] * r[1] + r[2] * r[2] + r[3] * r[3]);
      const float inv = scale / sqrtf(ss + d.l2_eps);
#pragma unroll
      for (int c = 0; c < 4; ++c) r[c] *= inv;
    }
    const size_t tg = (size_t)e.t0 + tb + i;
    *reinterpret_cast<float4*>(dst + (tg * nheads + head) * D + c0) = make_float4(r[0], r[1], r[2], r[3]);
  }
  if (u >= 2 * hq && lane < 8 && tb + lane < e.len) {
    const size_t tg = (size_t)e.t0 + tb + lane;
    g_out[tg * hv + head] = decay_gate_f(a[tg * hv + head], A_log[head], dt_bias[head]);
    beta_out[tg * hv + head] = sigmoid_f(b[tg * hv + head]);
  }
}

// ---- K5: gated RMSNorm epilogue ----------------------------------------------------------
// y = y_raw / sqrt(mean(y_raw^2) + eps) * norm_w * silu(z) per (token, value head) (field
// guide §02: RMS-normalise y, then gate with SiLU(z)).  One warp per EPI_ROWS consecutive
// rows, all loads issued first so the rows' memory latencies overlap.
constexpr int EPI_ROWS = 4;

template <bool IN_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(256) k_epilogue(Dims d, const float* __restrict__ y_raw,
                                                  const void* __restrict__ z,
                                                  const float* __restrict__ norm_w, void* __restrict__ y,
                                                  long rows) {
  const long row0 = ((long)blockIdx.x * 8 + (threadIdx.x >> 5)) * EPI_ROWS;
  if (row0 >= rows) return;
  const int c0 = (threadIdx.x & 31) * 4;
  float4 yr[EPI_ROWS], zz[EPI_ROWS];
#pragma unroll
  for (int r = 0; r < EPI_ROWS; ++r) {
    if (row0 + r < rows) {
      const size_t base = (size_t)(row0 + r) * D + c0;
      yr[r] = *reinterpret_cast<const float4*>(y_raw + base);
      zz[r] = load4<IN_BF16>(z, base);
    } else {
      yr[r] = zz[r] = make_float4(0, 0, 0, 0);
    }
  }
  const float4 nw = *reinterpret_cast<const float4*>(norm_w + c0);
  float ss[EPI_ROWS];
#pragma unroll
  for (int r = 0; r < EPI_ROWS; ++r) ss[r] = yr[r].x * yr[r].x + yr[r].y * yr[r].y + yr[r].z * yr[r].z + yr[r].w * yr[r].w;
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int r = 0; r < EPI_ROWS; ++r) ss[r] += __shfl_xor_sync(0xffffffffu, ss[r], o);
#pragma unroll
  for (int r = 0; r < EPI_ROWS; ++r) {
    if (row0 + r >= rows) break;
    const float inv = rsqrtf(ss[r] * (1.0f / D) + d.rms_eps);
    float4 o;
    o.x = yr[r].x * inv * nw.x * silu_fast(zz[r].x);
    o.y = yr[r].y * inv * nw.y * silu_fast(zz[r].y);
    o.z = yr[r].z * inv * nw.z * silu_fast(zz[r].z);
    o.w = yr[r].w * inv * nw.w * silu_fast(zz[r].w);
    store4<OUT_BF16>(y, (size_t)(row0 + r) * D + c0, o);
  }
}

}  // namespace gdn
