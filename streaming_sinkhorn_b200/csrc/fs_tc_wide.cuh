// fs_tc_wide.cuh -- the tensor-core passes for wide points (64 < d <= 1024, sm_100a).
//
// Same score as the d <= 64 passes (the attention form of the update, FlashSinkhorn summary,
// Methodology section 1; hi.hi + lo.hi + hi.lo fp16 MMAs into TMEM), but a 128-point tile of
// a wide image no longer fits shared memory next to its partner (512 d bytes each), so both
// operands stream through the stage ring in K-chunks of 64 coordinates: a stage holds one
// chunk of the row block and the same chunk of the key tile (2 x 32 KB), and the kc chunks
// of one key tile accumulate into one TMEM score tile. The key biases (and, for transport
// products, the key tile's payload) travel in a separate two-slot ring, kept until the
// epilogue (and the result MMA) are done with them.
//
// Wide images: per tile of 128 points, kc = d / 64 chunks of 32 KB, chunk-major; a chunk is
// [hi | lo] of its 64 coordinates in the core-matrix layout of the d = 64 images.
#pragma once

#include "fs_tc.cuh"

namespace fs {

constexpr int kTcChunk = 64;                                   // coordinates per K-chunk
constexpr uint32_t kTcChunkBytes = 128u * 2u * kTcChunk * 2u;  // one tile's chunk: 32 KB
constexpr int kTcWideMaxD = 1024;
constexpr int kTcWideStages = 3;  // potential passes: (row chunk, key chunk) pairs in flight
constexpr int kTcWideApplyStages = 2;

// Byte offset of element kk (< 128: [hi | lo] of chunk c) of point i in a wide image of kc
// chunks per point.
__host__ __device__ __forceinline__ int64_t tc_wide_offset(int64_t i, int c, int kk, int kc) {
  return ((i >> 7) * kc + c) * static_cast<int64_t>(kTcChunkBytes) +
         tc_image_offset(i & 127, kk, 2 * kTcChunk);
}

struct TcWideShape {
  static constexpr uint32_t STAGE_BYTES = 2u * kTcChunkBytes;  // row chunk, key chunk
  static constexpr uint32_t HY_BYTES = kTcCols * 4u;
  static constexpr uint32_t PAY_BYTES = 128u * 2u * kPayChannels * 2u;
  static constexpr uint32_t EX_BYTES = 1024u;                  // biases, padded
  static constexpr uint32_t EX_PAY_BYTES = PAY_BYTES + 1024u;  // payload + biases
  static constexpr size_t SMEM = kTcWideStages * STAGE_BYTES + 2u * EX_BYTES;
  static constexpr uint32_t P_BYTES = 128u * 128u * 2u;
  static constexpr size_t APPLY_SMEM =
      kTcWideApplyStages * STAGE_BYTES + 2u * P_BYTES + 2u * EX_PAY_BYTES;
  static_assert(SMEM <= kTcSmemBudget && APPLY_SMEM <= kTcSmemBudget, "shared memory");
};

// Producer role of the wide passes: for every key tile, its extras (biases, and the payload
// when pay_img is set) into slot t & 1, then its kc (row chunk, key chunk) pairs through
// the stage ring. Runs on one thread; on abort it lets its own copies land.
template <int ST>
__device__ __forceinline__ void tcw_produce(const TcParams& T, const unsigned char* pay_img,
                                            int64_t row0, int64_t t_begin, int n_tiles,
                                            unsigned char* sStage, unsigned char* sEx,
                                            uint32_t ex_bytes, uint64_t* full_bar,
                                            uint64_t* free_bar, uint64_t* ex_full,
                                            uint64_t* ex_free, volatile int* abort) {
  using W = TcWideShape;
  const int kc = T.kc;
  int q = 0, issued = 0;
  int ex_issued = 0;
  bool ok = true;
  for (int t = 0; ok && t < n_tiles; ++t) {
    const int e = t & 1;
    const int64_t kt = t_begin + t;
    if (t >= 2 && !tc_wait(&ex_free[e], static_cast<uint32_t>((t - 2) >> 1) & 1u, abort)) break;
    unsigned char* ex = sEx + e * ex_bytes;
    fence_proxy_async_smem();
    mbar_expect_tx(&ex_full[e], W::HY_BYTES + (pay_img ? W::PAY_BYTES : 0u));
    if (pay_img) bulk_g2s(ex, pay_img + kt * W::PAY_BYTES, W::PAY_BYTES, &ex_full[e]);
    bulk_g2s(ex + (pay_img ? W::PAY_BYTES : 0u), T.key_hy + kt * kTcCols, W::HY_BYTES,
             &ex_full[e]);
    ++ex_issued;
    for (int c = 0; c < kc; ++c, ++q) {
      const int s = q % ST;
      if (q >= ST && !tc_wait(&free_bar[s], static_cast<uint32_t>((q - ST) / ST) & 1u, abort)) {
        ok = false;
        break;
      }
      unsigned char* dst = sStage + s * W::STAGE_BYTES;
      fence_proxy_async_smem();
      mbar_expect_tx(&full_bar[s], W::STAGE_BYTES);
      bulk_g2s(dst, T.row_img + ((row0 >> 7) * kc + c) * kTcChunkBytes, kTcChunkBytes,
               &full_bar[s]);
      bulk_g2s(dst + kTcChunkBytes, T.key_img + (kt * kc + c) * kTcChunkBytes, kTcChunkBytes,
               &full_bar[s]);
      ++issued;
    }
  }
  if (*abort) {
    for (int u = (issued > ST ? issued - ST : 0); u < issued; ++u)
      (void)mbar_wait_bounded(&full_bar[u % ST], static_cast<uint32_t>(u / ST) & 1u);
    for (int u = (ex_issued > 2 ? ex_issued - 2 : 0); u < ex_issued; ++u)
      (void)mbar_wait_bounded(&ex_full[u & 1], static_cast<uint32_t>(u >> 1) & 1u);
  }
}

// The score tile t of the wide passes: kc chunks accumulated into accumulator tmem_s, each
// stage released by an MMA commit. Returns false on abort.
template <int ST>
__device__ __forceinline__ bool tcw_issue_tile(const TcParams& T, int& q, uint32_t tmem_s,
                                               unsigned char* sStage, uint64_t* full_bar,
                                               uint64_t* free_bar, uint32_t idesc,
                                               volatile int* abort) {
  using W = TcWideShape;
  for (int c = 0; c < T.kc; ++c, ++q) {
    const int s = q % ST;
    if (!tc_wait(&full_bar[s], static_cast<uint32_t>(q / ST) & 1u, abort)) return false;
    tc_fence_after();
    const uint32_t a0 = smem_u32(sStage + s * W::STAGE_BYTES);
    tc_issue_scores<kTcChunk>(tmem_s, a0, a0 + kTcChunkBytes, idesc, c > 0);
    tc_commit(&free_bar[s]);
  }
  return true;
}

// Potential-type pass (kPot, kMarg, kLse) for wide points.
__global__ void __launch_bounds__(kTcThreads, 1) lse_pass_tcw_kernel(const PassParams P,
                                                                    const TcParams T) {
  using W = TcWideShape;
  constexpr int ST = kTcWideStages;
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint64_t full_bar[ST], free_bar[ST];
  __shared__ uint64_t mma_bar[2], acc_free_bar[2];
  __shared__ uint64_t ex_full[2], ex_free[2];
  __shared__ uint64_t fin_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float2 merge[kTcGroups][kTcRows];

  unsigned char* sStage = smem;
  unsigned char* sEx = smem + ST * W::STAGE_BYTES;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kTcRows;
  const int split = blockIdx.y;
  const int64_t t_begin = static_cast<int64_t>(split) * T.tiles_per_split;
  int64_t t_end = t_begin + T.tiles_per_split;
  if (t_end > T.key_tiles) t_end = T.key_tiles;
  const int n_tiles = static_cast<int>(t_end - t_begin);
  volatile int* abort = &abort_sh;

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&free_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&mma_bar[b], 1);
      mbar_init(&acc_free_bar[b], kTcEpiWarps);
      mbar_init(&ex_full[b], 1);
      mbar_init(&ex_free[b], kTcEpiWarps);
    }
    mbar_init(&fin_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base_sh)),
                 "r"(kTcTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int quarter = warp & 3, grp = warp >> 2;
  const int r = quarter * 32 + lane;
  const int64_t i = row0 + r;
  TcRowLse rs = tc_row_lse_init((i < P.n_rows) ? P.kappa_f * T.row_nrm[i] : 0.0f);

  if (warp == kTcEpiWarps) {
    if (lane == 0)
      tcw_produce<ST>(T, nullptr, row0, t_begin, n_tiles, sStage, sEx, W::EX_BYTES, full_bar,
                      free_bar, ex_full, ex_free, abort);
  } else if (warp == kTcEpiWarps + 1) {
    if (lane == 0) {
      const uint32_t idesc = tc_instr_desc(kTcRows, kTcCols);
      int q = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int b = t & 1;
        if (t >= 2 && !tc_wait(&acc_free_bar[b], static_cast<uint32_t>((t - 2) >> 1) & 1u, abort))
          break;
        if (!tcw_issue_tile<ST>(T, q, tmem + static_cast<uint32_t>(b) * kTcCols, sStage, full_bar,
                                free_bar, idesc, abort))
          break;
        tc_commit(&mma_bar[b]);
      }
      // every MMA issued has completed once fin_bar fires: TMEM is never released under one
      tc_commit(&fin_bar);
      (void)mbar_wait_bounded(&fin_bar, 0);
    }
  } else {
    const u64 c2 = pk(T.c2, T.c2);
    for (int u = 0; u < n_tiles; ++u) {
      const int b = u & 1;
      const uint32_t ph = static_cast<uint32_t>(u >> 1) & 1u;
      if (!tc_wait(&mma_bar[b], ph, abort)) break;
      if (!tc_wait(&ex_full[b], ph, abort)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(b) * kTcCols + grp * kTcGC;
      float v[kTcGC];
#pragma unroll
      for (int c = 0; c < kTcGC; c += 32) tc_ld32_nowait(tbase + c, v + c);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free_bar[b]);
      tc_lse_tile(rs, v, reinterpret_cast<const float*>(sEx + b * W::EX_BYTES) + grp * kTcGC, c2);
      __syncwarp();
      if (lane == 0) mbar_arrive(&ex_free[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (abort_sh) {
    if (tid == 0) atomicOr(P.err, kErrTimeout);
  } else {
    tc_lse_finish<64>(P, merge, rs, warp < kTcEpiWarps, grp, r, i, split);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTcTmemCols));
}

// Transport apply pass (kApplyPay, kPayChannels channels) for wide points: the score tiles
// as above at the fixed row offsets, weights to shared memory, and the result MMA against
// the payload tile held in the extras slot of its key tile.
__global__ void __launch_bounds__(kTcThreads, 1)
    lse_apply_tcw_kernel(const PassParams P, const TcParams T, const TcApply A) {
  using W = TcWideShape;
  constexpr int ST = kTcWideApplyStages;
  constexpr int NC = kPayChannels;
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint64_t full_bar[ST], free_bar[ST];
  __shared__ uint64_t mma_bar[2], acc_free_bar[2];
  __shared__ uint64_t ex_full[2], ex_free[2];  // ex_free: 16 epilogue warps + the result MMA
  __shared__ uint64_t p_full[2], p_free[2];
  __shared__ uint64_t o_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float lsum[kTcGroups][kTcRows];

  unsigned char* sStage = smem;
  unsigned char* sP = smem + ST * W::STAGE_BYTES;
  unsigned char* sEx = sP + 2 * W::P_BYTES;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kTcRows;
  const int split = blockIdx.y;
  const int64_t t_begin = static_cast<int64_t>(split) * T.tiles_per_split;
  int64_t t_end = t_begin + T.tiles_per_split;
  if (t_end > T.key_tiles) t_end = T.key_tiles;
  const int n_tiles = static_cast<int>(t_end - t_begin);
  volatile int* abort = &abort_sh;

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&free_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&mma_bar[b], 1);
      mbar_init(&acc_free_bar[b], kTcEpiWarps);
      mbar_init(&ex_full[b], 1);
      mbar_init(&ex_free[b], kTcEpiWarps + 1);
      mbar_init(&p_full[b], kTcEpiWarps);
      mbar_init(&p_free[b], 1);
    }
    mbar_init(&o_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base_sh)),
                 "r"(kTcApplyTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tmem_o = tmem + 2u * kTcCols;
  const int quarter = warp & 3, grp = warp >> 2;
  const int r = quarter * 32 + lane;
  const int64_t i = row0 + r;
  u64 L = pk(0.0f, 0.0f);

  if (warp == kTcEpiWarps) {
    if (lane == 0)
      tcw_produce<ST>(T, A.pay_img, row0, t_begin, n_tiles, sStage, sEx, W::EX_PAY_BYTES,
                      full_bar, free_bar, ex_full, ex_free, abort);
  } else if (warp == kTcEpiWarps + 1) {
    if (lane == 0) {
      const uint32_t idesc_s = tc_instr_desc(kTcRows, kTcCols);
      const uint32_t idesc_o = tc_instr_desc(kTcRows, NC, true);
      constexpr uint32_t U_LO_OFF = (NC / 8) * kCoreLBO;
      int q = 0;
      for (int t = 0; t <= n_tiles; ++t) {
        if (t < n_tiles) {
          const int b = t & 1;
          if (t >= 2 && !tc_wait(&acc_free_bar[b], static_cast<uint32_t>((t - 2) >> 1) & 1u, abort))
            break;
          if (!tcw_issue_tile<ST>(T, q, tmem + static_cast<uint32_t>(b) * kTcCols, sStage,
                                  full_bar, free_bar, idesc_s, abort))
            break;
          tc_commit(&mma_bar[b]);
        }
        if (t >= 1) {
          const int u = t - 1, e = u & 1;
          const uint32_t ph = static_cast<uint32_t>(u >> 1) & 1u;
          if (!tc_wait(&p_full[e], ph, abort)) break;
          if (!tc_wait(&ex_full[e], ph, abort)) break;
          tc_fence_after();
          const uint32_t pa = smem_u32(sP + e * W::P_BYTES);
          const uint32_t ub = smem_u32(sEx + e * W::EX_PAY_BYTES);
#pragma unroll
          for (int s = 0; s < kTcCols / 16; ++s) {
            const uint64_t ad = tc_smem_desc(pa + s * 2u * kCoreLBO, kCoreLBO, kCoreSBO);
            const uint32_t ko = static_cast<uint32_t>(s) * 2u * kCoreSBO;
            tc_mma_f16(tmem_o, ad, tc_smem_desc(ub + ko, kCoreSBO, kCoreLBO), idesc_o,
                       (u > 0 || s > 0) ? 1u : 0u);
            tc_mma_f16(tmem_o, ad, tc_smem_desc(ub + U_LO_OFF + ko, kCoreSBO, kCoreLBO), idesc_o,
                       1u);
          }
          tc_commit(&p_free[e]);
          tc_commit(&ex_free[e]);
        }
      }
      tc_commit(&o_bar);
      (void)mbar_wait_bounded(&o_bar, 0);
    }
  } else {
    float off = 1.0e30f;  // padding rows: every weight is 0
    if (i < P.n_rows) off = P.kappa_f * T.row_nrm[i] + A.row_lse[i];
    const u64 c2 = pk(T.c2, T.c2);
    const u64 noff = pk(-off, -off);
    for (int u = 0; u < n_tiles; ++u) {
      const int b = u & 1;
      const uint32_t ph = static_cast<uint32_t>(u >> 1) & 1u;
      if (!tc_wait(&mma_bar[b], ph, abort)) break;
      if (!tc_wait(&ex_full[b], ph, abort)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(b) * kTcCols + grp * kTcGC;
      float v[kTcGC];
#pragma unroll
      for (int c = 0; c < kTcGC; c += 32) tc_ld32_nowait(tbase + c, v + c);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free_bar[b]);
      uint32_t h2[kTcGC / 2];
      tc_weights_tile(v,
                      reinterpret_cast<const float*>(sEx + b * W::EX_PAY_BYTES + W::PAY_BYTES) +
                          grp * kTcGC,
                      c2, noff, L, h2);
      __syncwarp();
      if (lane == 0) mbar_arrive(&ex_free[b]);  // its biases have been read
      if (u >= 2 && !tc_wait(&p_free[b], static_cast<uint32_t>((u - 2) >> 1) & 1u, abort)) break;
      tc_store_weights(sP + b * W::P_BYTES, r, grp, h2);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  {
    float l0, l1;
    upk(L, l0, l1);
    if (warp < kTcEpiWarps) lsum[grp][r] = l0 + l1;
  }
  __syncthreads();
  if (abort_sh) {
    if (tid == 0) atomicOr(P.err, kErrTimeout);
  } else if (warp < 8) {
    const int half = grp;  // the first two column groups read NC / 2 channels each
    if (mbar_wait_bounded(&o_bar, 0)) {
      tc_fence_after();
      constexpr int NH = NC / 2;
      float o[NH];
      const uint32_t obase = tmem_o + (static_cast<uint32_t>(quarter * 32) << 16) + half * NH;
#pragma unroll
      for (int c = 0; c < NH; c += 8) tc_ld8_nowait(obase + c, o + c);
      tc_wait_ld();
      double l = 0.0;
#pragma unroll
      for (int qq = 0; qq < kTcGroups; ++qq) l += static_cast<double>(lsum[qq][r]);
      const double inv = static_cast<double>(*A.pay_inv_scale);
      if (i < P.n_rows) {
        if (P.n_splits == 1) {
#pragma unroll
          for (int c = 0; c < NH; ++c)
            tc_apply_finish<kApplyPay>(P, A, i, half * NH + c, static_cast<double>(o[c]) * inv, l);
        } else {
          const int64_t ps = static_cast<int64_t>(split);
          if (half == 0) P.part_l[ps * P.rows_pad + i] = static_cast<float>(l);
#pragma unroll
          for (int c = 0; c < NH; ++c)
            P.part_a[(ps * NC + half * NH + c) * P.rows_pad + i] =
                static_cast<float>(static_cast<double>(o[c]) * inv);
        }
      }
    } else {
      atomicOr(P.err, kErrTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTcApplyTmemCols));
}

// ---- preparation for the wide passes -------------------------------------------------------

// The wide image of one cloud (centred on ctr, scaled, [hi | lo] per 64-coordinate chunk)
// and its centred squared norms, for all padded points; kc chunks per point.
__global__ void __launch_bounds__(256) build_wide_image_kernel(const float* pts, int64_t count,
                                                               int32_t d_real, int32_t kc,
                                                               const double* ctr, float scale,
                                                               unsigned char* img, float* nrm,
                                                               int64_t count_pad) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count_pad) return;
  double n2 = 0.0;
  for (int k = 0; k < kc * kTcChunk; ++k) {
    float u = 0.0f;
    if (i < count && k < d_real) {
      const double c = static_cast<double>(pts[i * d_real + k]) - ctr[k];
      n2 += c * c;
      u = static_cast<float>(c * scale);
    }
    const __half hi = __float2half_rn(u);
    const __half lo = __float2half_rn(u - __half2float(hi));
    const int c = k / kTcChunk, kk = k % kTcChunk;
    *reinterpret_cast<__half*>(img + tc_wide_offset(i, c, kk, kc)) = hi;
    *reinterpret_cast<__half*>(img + tc_wide_offset(i, c, kTcChunk + kk, kc)) = lo;
  }
  nrm[i] = static_cast<float>(n2);
}

// grad_i = 2 (w_i x_i - (P y)_i): the envelope gradient from the transport product P y at
// the plan of (F(g), g) (rows sum to w).
__global__ void __launch_bounds__(256) grad_from_py_kernel(const float* x, const float* w,
                                                           float w_uniform, const float* py,
                                                           int64_t n, int32_t d, float* grad) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n * d) return;
  const int64_t i = t / d;
  const double wi = w ? static_cast<double>(w[i]) : static_cast<double>(w_uniform);
  grad[t] = static_cast<float>(2.0 * (wi * static_cast<double>(x[t]) - static_cast<double>(py[t])));
}

}  // namespace fs
