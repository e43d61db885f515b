// fs_tc.cuh -- the streaming pass for d > 16 on the tcgen05 tensor cores (sm_100a).
//
// For wide points the score is a real contraction, so the pass uses the attention form of
// the update (FlashSinkhorn summary, Methodology section 1): with the clouds centred,
//     z_ij = hy_j + 2 kappa x_i.y_j - kappa |x_i|^2,    hy_j = H_j - kappa |y_j|^2,
// and x.y is computed by the tensor cores for a 128-row block against 128-column key
// tiles. To keep float32-level accuracy the inputs are scaled by a power of two s and
// split into fp16 halves, u = hi + lo (hi = fp16(u), lo = fp16(u - hi)); the MMA takes
//     A = [hi_x | lo_x | hi_x],  B = [hi_y | hi_y | lo_y]   (K = 3D),
// so one K = 3D product gives hi.hi + lo.hi + hi.lo = s^2 x.y up to ~2^-22 relative, with
// fp32 accumulation in tensor memory.
//
// Operand images. Each cloud is stored twice in global memory (as rows with the A order,
// as keys with the B order), already in the shared-memory layout the MMA reads: per tile of
// 128 points, 8x8-element core matrices (8 points x 16 bytes of K) stored K-block-major,
// core(g, kb) at byte (kb * 16 + g) * 128. A K-step of 16 elements is two consecutive
// K-blocks (leading-byte offset 16 * 128 B); consecutive 8-point groups are 128 B apart
// (stride-byte offset). A tile is therefore one contiguous block that a single TMA bulk copy
// moves into shared memory.
//
// Kernel: one CTA per 128-row block and column split, 10 warps with fixed roles. Warp 8
// streams key tiles (B image + hy) through a 3-stage ring with TMA bulk copies; warp 9
// issues the MMAs of tile t into one of two TMEM accumulators; warps 0-7 run the online
// max/sum (warp w reads TMEM lanes 32 (w % 4) .. +31, the columns of half w / 4 of each
// tile). Roles hand off through mbarriers only: a tile's stage is free once its MMAs have
// completed (tcgen05.commit) and the 8 epilogue warps have read its biases; an accumulator
// is free once the 8 epilogue warps have loaded it. No CTA barrier runs per tile.
#pragma once

#include <cuda_fp16.h>
#include "fs_kernels.cuh"

namespace fs {

constexpr int kTcRows = 128;     // rows per CTA (MMA M)
constexpr int kTcCols = 128;     // key columns per tile (MMA N)
constexpr int kTcStages = 3;
constexpr int kTcEpiWarps = 8;  // epilogue warps: 4 TMEM lane quarters x 2 column halves
constexpr int kTcThreads = (kTcEpiWarps + 2) * 32;  // + a producer warp and an MMA warp
constexpr uint32_t kTcTmemCols = 256;  // two accumulators of kTcCols fp32 columns

template <int D>
struct TcShape {
  static constexpr int K = 3 * D;                  // split-operand K extent
  static constexpr int KSTEPS = K / 16;            // MMA K = 16 for fp16
  static constexpr uint32_t TILE_BYTES = 128u * K * 2u;
  static constexpr uint32_t HY_BYTES = kTcCols * 4u;
  static constexpr uint32_t STAGE_BYTES = TILE_BYTES + 1024u;  // hy, padded to keep stages aligned
  static constexpr uint32_t LBO = 16u * 128u;      // next K-block (second half of a K-step)
  static constexpr uint32_t SBO = 128u;            // next 8-point group
  static constexpr size_t SMEM = static_cast<size_t>(TILE_BYTES) + kTcStages * STAGE_BYTES;
};

// Byte offset of K element kk of point i in an operand image with K elements per point.
__host__ __device__ __forceinline__ int64_t tc_image_offset(int64_t i, int kk, int K) {
  const int64_t tile = i >> 7;
  const int r = static_cast<int>(i & 127);
  return tile * (128ll * K * 2) + (static_cast<int64_t>(kk >> 3) * 16 + (r >> 3)) * 128 +
         (r & 7) * 16 + (kk & 7) * 2;
}

// Shared-memory matrix descriptor: K-major, no swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t tc_smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Instruction descriptor of kind::f16: fp16 A and B (K-major), fp32 accumulate, M x N.
__host__ __device__ constexpr uint32_t tc_instr_desc(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane; the caller waits (tcgen05.wait::ld).
__device__ __forceinline__ void tc_ld32_nowait(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

struct TcParams {
  const unsigned char* row_img;  // query cloud as rows (A order), tiles of 128 points
  const unsigned char* key_img;  // streamed cloud as keys (B order)
  const float* key_hy;           // hy of the streamed cloud, padded to whole tiles
  const float* row_nrm;          // |x_i|^2 of the query cloud (centred)
  int64_t key_tiles;             // tiles of 128 keys
  int64_t tiles_per_split;
  float c2;                      // 2 kappa / s^2: scale of the MMA result
};

// Waits for phase `parity` of `bar`, giving up after kWaitLimitNs or as soon as another
// role of the CTA has raised `abort`.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) lse_pass_tc_kernel(const PassParams P,
                                                                   const TcParams T) {
  using S = TcShape<D>;
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint64_t full_bar[kTcStages];   // tile landed (producer's expect_tx)
  __shared__ uint64_t free_bar[kTcStages];   // stage reusable: MMA commit + 8 epilogue warps
  __shared__ uint64_t mma_bar[2];            // accumulator ready (MMA commit)
  __shared__ uint64_t acc_free_bar[2];       // accumulator read by the 8 epilogue warps
  __shared__ uint64_t a_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float2 merge[kTcRows];

  unsigned char* sA = smem;
  unsigned char* sStage = smem + S::TILE_BYTES;
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
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&free_bar[s], kTcEpiWarps + 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&mma_bar[b], 1);
      mbar_init(&acc_free_bar[b], kTcEpiWarps);
    }
    mbar_init(&a_bar, 1);
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

  float m = -INFINITY;  // epilogue row state (origin-free running offset) ...
  u64 L = pk(0.0f, 0.0f);
  const int quarter = warp & 3, half = (warp >> 2) & 1;
  const int r = quarter * 32 + lane;
  const int64_t i = row0 + r;

  if (warp == kTcEpiWarps) {
    // ---- producer: the row block once, then key tiles through the stage ring ----------
    if (lane == 0) {
      int issued = 0, waited_free = 0;
      mbar_expect_tx(&a_bar, S::TILE_BYTES);
      bulk_g2s(sA, T.row_img + (row0 >> 7) * S::TILE_BYTES, S::TILE_BYTES, &a_bar);
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % kTcStages;
        if (t >= kTcStages) {
          if (!tc_wait(&free_bar[st], static_cast<uint32_t>((t - kTcStages) / kTcStages) & 1u, abort))
            break;
          ++waited_free;
        }
        unsigned char* dst = sStage + st * S::STAGE_BYTES;
        const int64_t kt = t_begin + t;
        fence_proxy_async_smem();
        mbar_expect_tx(&full_bar[st], S::TILE_BYTES + S::HY_BYTES);
        bulk_g2s(dst, T.key_img + kt * S::TILE_BYTES, S::TILE_BYTES, &full_bar[st]);
        bulk_g2s(dst + S::TILE_BYTES, T.key_hy + kt * kTcCols, S::HY_BYTES, &full_bar[st]);
        ++issued;
      }
      (void)waited_free;
      // Copies never waited for by the MMA role: let them land before the CTA exits.
      if (*abort) {
        (void)mbar_wait_bounded(&a_bar, 0);
        for (int t = (issued > kTcStages ? issued - kTcStages : 0); t < issued; ++t)
          (void)mbar_wait_bounded(&full_bar[t % kTcStages], static_cast<uint32_t>(t / kTcStages) & 1u);
      }
    }
  } else if (warp == kTcEpiWarps + 1) {
    // ---- MMA issuer: tile t into accumulator t & 1 --------------------------------------
    if (lane == 0) {
      const uint32_t idesc = tc_instr_desc(kTcRows, kTcCols);
      int committed = 0;
      bool ok = tc_wait(&a_bar, 0, abort);
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int st = t % kTcStages, b = t & 1;
        if (!tc_wait(&full_bar[st], static_cast<uint32_t>(t / kTcStages) & 1u, abort)) break;
        if (t >= 2 && !tc_wait(&acc_free_bar[b], static_cast<uint32_t>((t - 2) >> 1) & 1u, abort))
          break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA);
        const uint32_t b0 = smem_u32(sStage + st * S::STAGE_BYTES);
        const uint32_t d = tmem + static_cast<uint32_t>(b) * kTcCols;
#pragma unroll
        for (int s = 0; s < S::KSTEPS; ++s) {
          tc_mma_f16(d, tc_smem_desc(a0 + s * 2 * S::LBO, S::LBO, S::SBO),
                     tc_smem_desc(b0 + s * 2 * S::LBO, S::LBO, S::SBO), idesc, s > 0 ? 1u : 0u);
        }
        tc_commit(&mma_bar[b]);
        tc_commit(&free_bar[st]);
        ++committed;
      }
      // On abort, let the MMAs already issued finish before TMEM is released.
      if (*abort && committed > 0)
        (void)mbar_wait_bounded(&mma_bar[(committed - 1) & 1],
                                static_cast<uint32_t>((committed - 1) >> 1) & 1u);
    }
  } else {
    // ---- epilogue warps: online max/sum of one row over half of every tile ------------
    const float knrm = (i < P.n_rows) ? P.kappa_f * T.row_nrm[i] : 0.0f;
    float base = 0.0f, mo = knrm;
    const u64 c2 = pk(T.c2, T.c2);
    for (int u = 0; u < n_tiles; ++u) {
      const int b = u & 1, st = u % kTcStages;
      if (!tc_wait(&mma_bar[b], static_cast<uint32_t>(u >> 1) & 1u, abort)) break;
      tc_fence_after();
      const float* hy = reinterpret_cast<const float*>(sStage + st * S::STAGE_BYTES + S::TILE_BYTES);
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(b) * kTcCols + half * 64;
      float v[64];
      tc_ld32_nowait(tbase, v);
      tc_ld32_nowait(tbase + 32, v + 32);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free_bar[b]);
      const u64* hv = reinterpret_cast<const u64*>(hy + half * 64);
      u64 tv[32];
      const u64 nmo = pk(-mo, -mo);
#pragma unroll
      for (int j = 0; j < 32; ++j) tv[j] = add2(fma2(c2, pk(v[2 * j], v[2 * j + 1]), hv[j]), nmo);
      __syncwarp();
      if (lane == 0) mbar_arrive(&free_bar[st]);
      float a0, a1;
      upk(tv[0], a0, a1);
      float mx = fmaxf(a0, a1);
#pragma unroll
      for (int j = 1; j < 32; ++j) {
        upk(tv[j], a0, a1);
        mx = max3(mx, a0, a1);
      }
      const float mx_abs = mx + base;
      if (mx_abs > m + kLazyThr && mx > kEmptyCut) {
        const float sc = ex2(m - mx_abs);
        L = mul2(L, pk(sc, sc));
        const u64 sh = pk(-mx, -mx);
#pragma unroll
        for (int j = 0; j < 32; ++j) tv[j] = add2(tv[j], sh);
        m = mx_abs;
        base = mx_abs;
        mo = knrm + m;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float t0, t1;
        upk(tv[j], t0, t1);
        L = add2(L, pk(ex2(t0), ex2(t1)));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (abort_sh) {
    if (tid == 0) atomicOr(P.err, kErrTimeout);
  } else {
    // Merge the two column halves of each row, then finish the row.
    float l0, l1;
    upk(L, l0, l1);
    if (warp < kTcEpiWarps && half == 1) merge[r] = make_float2(m, l0 + l1);
    __syncthreads();
    double dev = 0.0, mass = 0.0;
    if (warp < kTcEpiWarps && half == 0 && i < P.n_rows) {
      const float2 o = merge[r];
      const float mm = fmaxf(m, o.x);
      float l = 0.0f;
      if (m != -INFINITY) l += (l0 + l1) * ex2(m - mm);
      if (o.x != -INFINITY) l += o.y * ex2(o.x - mm);
      if (P.n_splits == 1) {
        const double lse2 = static_cast<double>(mm) + log2(static_cast<double>(l));
        if (P.kind == kPot) {
          finish_pot<D>(P, i, lse2);
        } else {
          finish_marg(P, i, lse2, dev, mass);
        }
      } else {
        const int64_t o2 = static_cast<int64_t>(split) * P.rows_pad + i;
        P.part_m[o2] = mm;
        P.part_l[o2] = l;
      }
    }
    if (P.n_splits == 1 && P.kind == kMarg) block_reduce_marg(dev, dev, mass, P.acc);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTcTmemCols));
}

// ---- preparation for the tensor-core pass -----------------------------------------------

// Per-coordinate sums (float64) and the largest |coordinate| of one cloud.
__global__ void __launch_bounds__(256) coord_stats_kernel(const float* pts, int64_t count,
                                                          int32_t d, double* sums,
                                                          unsigned* maxabs_bits) {
  const int k = blockIdx.y;
  double s = 0.0;
  float mx = 0.0f;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < count;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = pts[j * d + k];
    s += v;
    mx = fmaxf(mx, fabsf(v));
  }
  s = warp_sum(s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&sums[k], s);
    atomicMax(maxabs_bits, __float_as_uint(mx));  // order-preserving for mx >= 0
  }
}

struct TcCenter {
  double c[64];
};

// Both operand images of one cloud and its centred squared norms, for all padded points.
template <int D>
__global__ void __launch_bounds__(256) build_images_kernel(const float* pts, int64_t count,
                                                           int32_t d_real, const TcCenter ctr,
                                                           float scale, unsigned char* row_img,
                                                           unsigned char* key_img, float* nrm,
                                                           int64_t count_pad) {
  constexpr int K = 3 * D;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count_pad) return;
  double n2 = 0.0;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    float u = 0.0f;
    if (i < count && k < d_real) {
      const double c = static_cast<double>(pts[i * d_real + k]) - ctr.c[k];
      n2 += c * c;
      u = static_cast<float>(c * scale);
    }
    const __half hi = __float2half_rn(u);
    const __half lo = __float2half_rn(u - __half2float(hi));
    *reinterpret_cast<__half*>(row_img + tc_image_offset(i, k, K)) = hi;
    *reinterpret_cast<__half*>(row_img + tc_image_offset(i, D + k, K)) = lo;
    *reinterpret_cast<__half*>(row_img + tc_image_offset(i, 2 * D + k, K)) = hi;
    *reinterpret_cast<__half*>(key_img + tc_image_offset(i, k, K)) = hi;
    *reinterpret_cast<__half*>(key_img + tc_image_offset(i, D + k, K)) = hi;
    *reinterpret_cast<__half*>(key_img + tc_image_offset(i, 2 * D + k, K)) = lo;
  }
  nrm[i] = static_cast<float>(n2);
}

// hy_j = kappa pot_j + log2 w_j - kappa |y_j|^2 for real points (pot = 0 if NULL); padding
// columns get kLogZero.
__global__ void __launch_bounds__(256) tc_key_bias_kernel(float* hy, int64_t count,
                                                          int64_t count_pad, const float* pot,
                                                          const float* lw, const float* nrm,
                                                          double kappa) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= count_pad) return;
  if (j >= count) {
    hy[j] = kLogZero;
    return;
  }
  const double p = pot ? static_cast<double>(pot[j]) : 0.0;
  hy[j] = static_cast<float>(kappa * p + static_cast<double>(lw[j]) -
                             kappa * static_cast<double>(nrm[j]));
}

}  // namespace fs
