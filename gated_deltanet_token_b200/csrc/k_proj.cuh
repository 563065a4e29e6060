// k_proj.cuh -- the projections on either side of the mixer as tcgen05 GEMMs (bf16 operands,
// fp32 accumulation in tensor memory).
//
//   input projection  ("Qwen3.8-Flash-Next" technical report, Fig. 2: the projected query, key
//   and value streams): [q | k | v | z | a | b] = x W_in^T for the block input x [T][hidden];
//   output projection (field guide §02: RMS-normalise y, gate with SiLU(z), output projection):
//   out = y W_out^T for the gated mixer output y [T][h_v d_v].
//
// C[m][n] = sum_k A[m][k] B[n][k]: A = the activations [M][K], B = the weights [N][K] (the
// nn.Linear layout), both K-major bf16.  C is cut into 128 x 256 tiles; a persistent CTA (one
// per SM) takes every gridDim.x-th tile:
//   warp 0, one lane: tensor copies (TMA, 128-byte swizzle) of 64-wide K blocks of A (128 rows,
//                      16 KB) and B (256 rows, 32 KB) into a 4-stage ring that runs on across tiles;
//   warp 1, one lane: the MMAs, four 128 x 256 x 16 tcgen05.mma per K block, accumulating in one
//                      of two 256-column halves of tensor memory (alternating by tile); each stage
//                      is handed back to the producer by tcgen05.commit;
//   warps 2..5:       the epilogue -- TMEM rows to registers, then each 32-column group goes to
//                      the output segment it belongs to (bf16 round-to-nearest-even, or fp32); then
//                      the accumulator half is handed back to the MMA lane.
// Rows past M and columns past N are zero-filled by the copies and not stored.  Every wait is
// bounded (a timeout records GDN_ERR_DEVICE_TIMEOUT and the CTA leaves after its copies landed).
#pragma once
#include <cuda.h>

#include "gdn_common.cuh"
#include "tc_ptx.cuh"

namespace gdn {

constexpr int PJ_BM = 128, PJ_BN = 256, PJ_BK = 64, PJ_STAGES = 4;
constexpr uint32_t PJ_A_BYTES = PJ_BM * PJ_BK * 2;  // 16 KB
constexpr uint32_t PJ_B_BYTES = PJ_BN * PJ_BK * 2;  // 32 KB
constexpr uint32_t PJ_STAGE_BYTES = PJ_A_BYTES + PJ_B_BYTES;
constexpr size_t PJ_SMEM = (size_t)PJ_STAGES * PJ_STAGE_BYTES + 1024;  // + alignment slack
constexpr int PJ_MAX_SEGS = 6;

// A run of output columns [n0, n1) stored at out + row * ld + (n - n0), bf16 or fp32.
struct ProjSeg {
  int n0, n1;
  long long ld;  // elements per row
  int f32;
  void* out;
};
struct ProjOut {
  int nseg;
  ProjSeg seg[PJ_MAX_SEGS];
};

namespace tc {
// 2-D tiled tensor copy global -> shared (no multicast), completion counted in bytes on `bar`.
// x (the K coordinate, in elements) must be a multiple of 8 for bf16.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// Shared-memory matrix descriptor of a K-major tile in the 128-byte swizzled layout that the
// tensor copies produce: rows of 128 bytes (64 bf16 of K), 8-row groups 1024 bytes apart (SBO),
// descriptor version 1 (sm_100), layout type 2 (128-byte swizzle).  The tile base is 1024-byte
// aligned; the k-th 16-wide K slice starts 32 k bytes further (the swizzle is a function of the
// address bits, so the same descriptor form addresses it).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;              // leading byte offset: unused for swizzled K-major tiles
  d |= (uint64_t)(1024u >> 4) << 32;    // stride byte offset: 8 rows x 128 bytes
  d |= (uint64_t)1u << 46;              // descriptor version for sm_100
  d |= (uint64_t)2u << 61;              // 128-byte swizzle
  return d;
}
}  // namespace tc

// Stores one 32-column group of accumulator row m (columns n .. n + 31, values r[0..31]) into
// the output segments.
__device__ __forceinline__ void proj_store_group(const ProjOut& po, int m, int n, int N, const uint32_t (&r)[32]) {
  int si = 0;
  while (si + 1 < po.nseg && n >= po.seg[si].n1) ++si;
  if (n + 32 > po.seg[si].n1 && si + 1 < po.nseg) {  // the group crosses into the next segment
    for (int i = 0; i < 32 && n + i < N; ++i) {
      int sj = si;
      while (sj + 1 < po.nseg && n + i >= po.seg[sj].n1) ++sj;
      const ProjSeg g = po.seg[sj];
      const long long off = (long long)m * g.ld + (n + i - g.n0);
      if (g.f32) static_cast<float*>(g.out)[off] = __uint_as_float(r[i]);
      else static_cast<uint16_t*>(g.out)[off] = f2bf(__uint_as_float(r[i]));
    }
    return;
  }
  const ProjSeg sg = po.seg[si];
  const int nn = n - sg.n0, cnt = min(32, sg.n1 - n);
  if (sg.f32) {
    float* o = static_cast<float*>(sg.out) + (long long)m * sg.ld + nn;
    if (cnt == 32 && ((reinterpret_cast<uintptr_t>(o) & 15u) == 0)) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<float4*>(o)[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                      __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
    } else {
      for (int i = 0; i < cnt; ++i) o[i] = __uint_as_float(r[i]);
    }
  } else {
    uint16_t* o = static_cast<uint16_t*>(sg.out) + (long long)m * sg.ld + nn;
    if (cnt == 32 && ((reinterpret_cast<uintptr_t>(o) & 15u) == 0)) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const __nv_bfloat162 b2 =
              __floats2bfloat162_rn(__uint_as_float(r[8 * i + 2 * u]), __uint_as_float(r[8 * i + 2 * u + 1]));
          w[u] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        reinterpret_cast<uint4*>(o)[i] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      for (int i = 0; i < cnt; ++i) o[i] = f2bf(__uint_as_float(r[i]));
    }
  }
}

// Persistent: CTA b takes tiles b, b + gridDim.x, ... (tile t: rows 128 (t % tiles_m), columns
// 256 (t / tiles_m)).  The copy ring runs on across tiles, and the accumulator alternates
// between two 256-column halves of tensor memory, so one tile's epilogue overlaps the next
// tile's MMAs.
__global__ void __launch_bounds__(192, 1) k_proj_gemm(int M, int N, int K, const __grid_constant__ CUtensorMap tm_a,
                                                      const __grid_constant__ CUtensorMap tm_b, ProjOut po) {
  extern __shared__ __align__(1024) uint8_t pj_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = K / PJ_BK;
  const int tiles_m = (M + PJ_BM - 1) / PJ_BM, tiles_n = (N + PJ_BN - 1) / PJ_BN, ntiles = tiles_m * tiles_n;
  // the swizzled tiles need 1024-byte aligned bases
  const uint32_t base_u = (tc::smem_u32(pj_raw) + 1023u) & ~1023u;
  __shared__ uint64_t full[PJ_STAGES], empty[PJ_STAGES], acc_full[2], acc_empty[2];
  __shared__ uint32_t tslot;
  __shared__ int s_abort;
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < PJ_STAGES; ++s) {
      tc::mbar_init(tc::smem_u32(&full[s]), 1);
      tc::mbar_init(tc::smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(tc::smem_u32(&acc_full[b]), 1);
      tc::mbar_init(tc::smem_u32(&acc_empty[b]), 4);  // one lane of each epilogue warp
    }
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(&tslot), 2 * PJ_BN);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tslot;
  auto stage_a = [&](int s) { return base_u + (uint32_t)s * PJ_STAGE_BYTES; };
  auto stage_b = [&](int s) { return base_u + (uint32_t)s * PJ_STAGE_BYTES + PJ_A_BYTES; };
  auto fail = [&]() {
    s_abort = 1;
    atomicExch(&g_gdn_status, -7);
  };
  auto aborted = [&]() { return *static_cast<volatile int*>(&s_abort) != 0; };
  // bounded wait; once any thread recorded a timeout, a wait that does not complete at its
  // first try returns false at once
  auto wait_ok = [&](uint64_t& bar, uint32_t parity) -> bool {
    if (tc::mbar_try_wait(tc::smem_u32(&bar), parity)) return true;
    if (aborted()) return false;
    if (tc::mbar_wait(tc::smem_u32(&bar), parity)) return true;
    fail();
    return false;
  };
  int issued = 0;  // (producer) K blocks whose copies were issued, over all tiles
  if (warp == 0 && lane == 0) {
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const int m0 = (t % tiles_m) * PJ_BM, n0 = (t / tiles_m) * PJ_BN;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = issued % PJ_STAGES;
        if (issued >= PJ_STAGES && !wait_ok(empty[s], (uint32_t)((issued / PJ_STAGES) - 1) & 1u)) {
          ok = false;
          break;
        }
        const uint32_t bar = tc::smem_u32(&full[s]);
        tc::mbar_arrive_expect_tx(bar, PJ_STAGE_BYTES);
        tc::tma_load_2d(stage_a(s), &tm_a, kb * PJ_BK, m0, bar);
        tc::tma_load_2d(stage_b(s), &tm_b, kb * PJ_BK, n0, bar);
        ++issued;
      }
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = tc::idesc_bf16(PJ_BM, PJ_BN, 0, 0);
    int it = 0, lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++lt) {
      const int b = lt & 1;
      // the epilogue has drained this accumulator (tile lt - 2)
      if (lt >= 2 && !wait_ok(acc_empty[b], (uint32_t)((lt >> 1) - 1) & 1u)) break;
      tc::tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(b * PJ_BN);
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = it % PJ_STAGES;
        if (!wait_ok(full[s], (uint32_t)(it / PJ_STAGES) & 1u)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint64_t da = tc::sdesc_sw128(stage_a(s)), db = tc::sdesc_sw128(stage_b(s));
#pragma unroll
        for (int kk = 0; kk < PJ_BK / 16; ++kk)
          tc::umma_bf16(acc, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), idesc, (kb | kk) != 0);
        tc::umma_commit(tc::smem_u32(&empty[s]));  // the stage is free once these MMAs have read it
      }
      if (ok) tc::umma_commit(tc::smem_u32(&acc_full[b]));
    }
  } else if (warp >= 2) {
    // epilogue: warp w holds TMEM lanes 32 (w % 4) .. + 31, i.e. rows m0 + 32 (w % 4) + lane
    const int q4 = warp & 3;
    int lt = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
      const int b = lt & 1;
      const int m0 = (t % tiles_m) * PJ_BM, n0 = (t / tiles_m) * PJ_BN, m = m0 + q4 * 32 + lane;
      // warp-uniform, so that the warp-collective TMEM loads run on every lane or none
      if (!__all_sync(0xffffffffu, wait_ok(acc_full[b], (uint32_t)(lt >> 1) & 1u))) break;
      tc::tc_fence_after();
      const uint32_t acc = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(b * PJ_BN);
#pragma unroll 1
      for (int cc = 0; cc < PJ_BN / 32 && n0 + cc * 32 < N; ++cc) {  // warp-uniform bound
        uint32_t r[32];
        __syncwarp();
        tc::tmem_ld32(acc + cc * 32, r);  // the whole warp loads
        tc::tmem_wait_ld();
        if (m < M) proj_store_group(po, m, n0 + cc * 32, N, r);
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tc::smem_u32(&acc_empty[b]));  // this accumulator may be reused
    }
  }
  // after a timeout, the copies issued must land before the shared memory is released: each
  // stage's last arming completes its phase
  if (warp == 0 && lane == 0 && aborted()) {
    for (int kb = issued - PJ_STAGES < 0 ? 0 : issued - PJ_STAGES; kb < issued; ++kb)
      (void)tc::mbar_wait(tc::smem_u32(&full[kb % PJ_STAGES]), (uint32_t)(kb / PJ_STAGES) & 1u);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 2 * PJ_BN);
}

}  // namespace gdn
