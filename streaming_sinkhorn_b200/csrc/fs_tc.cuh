// fs_tc.cuh -- the streaming passes for d > 16 on the tcgen05 tensor cores (sm_100a).
//
// For wide points the score is a real contraction, so the passes use the attention form of
// the update (FlashSinkhorn summary, Methodology section 1): with the clouds centred,
//     z_ij = hy_j + 2 kappa x_i.y_j - kappa |x_i|^2,    hy_j = H_j - kappa |y_j|^2,
// and x.y is computed by the tensor cores for a 128-row block against 128-column key
// tiles. To keep float32-level accuracy the inputs are scaled by a power of two s and
// split into fp16 halves, u = hi + lo (hi = fp16(u), lo = fp16(u - hi)); each 16-wide
// K-step issues three MMAs, hi_x.hi_y + lo_x.hi_y + hi_x.lo_y = s^2 x.y up to ~2^-22
// relative, with fp32 accumulation in tensor memory.
//
// Operand images. Each cloud is stored once in global memory as [hi | lo] (K = 2D fp16 per
// point), already in the shared-memory layout the MMA reads: per tile of 128 points,
// 8x8-element core matrices (8 points x 16 bytes of K) stored K-block-major, core(g, kb) at
// byte (kb * 16 + g) * 128. For the score MMA (points along M or N, coordinates along K)
// that is the K-major layout: a K-step of 16 elements is two consecutive K-blocks
// (leading-byte offset 16 * 128 B), consecutive 8-point groups are 128 B apart (stride-byte
// offset). Read the other way (points along K, coordinates along N) the same bytes are the
// MN-major layout: 8 consecutive points of one core matrix are 16-byte rows, the next 8
// points are 128 B on (leading-byte offset), the next 8 coordinates 16 * 128 B on
// (stride-byte offset). The apply pass uses it so as the B operand of sum_j p_ij y_j. A
// tile is one contiguous block that a single TMA bulk copy moves into shared memory.
//
// Potential pass (lse_pass_tc_kernel): one CTA per 128-row block and column split, 18 warps
// with fixed roles. Warp 16 streams key tiles (image + hy) through a 3-stage ring with TMA
// bulk copies; warp 17 issues the MMAs of tile t into one of two TMEM accumulators; warps
// 0-15 run the online max/sum (warp w reads TMEM lanes 32 (w % 4) .. +31, the 32 columns of
// group w / 4 of each tile: sixteen warps keep enough exponentials in flight for the MUFU
// unit). Roles hand off through mbarriers only.
//
// Apply pass (lse_apply_tc_kernel, FlashSinkhorn summary, section 3, "Transport Matrix
// Application"): out_i = sum_j p_ij U_j / sum_j p_ij with p_ij = 2^(z_ij - LSE2_i), the
// offset LSE2_i taken from a potential-type pass run just before (so p <= 1, no running
// rescale of a TMEM accumulator is needed). The epilogue writes 2^15 p as fp16 into a
// shared-memory weight tile, the MMA warp multiplies it by the key tile's U (the key
// coordinates for the gradient, a payload image for transport products), hi and lo halves,
// into a third TMEM accumulator, and the epilogue sums the same rounded weights, so the
// result is an exact convex combination of U up to fp16 weight rounding.
#pragma once

#include <cuda_fp16.h>
#include "fs_kernels.cuh"

namespace fs {

constexpr int kTcRows = 128;     // rows per CTA (MMA M)
constexpr int kTcCols = 128;     // key columns per tile (MMA N of the score)
constexpr int kTcStages = 3;
constexpr int kTcEpiWarps = 16;  // epilogue warps: 4 TMEM lane quarters x 4 column groups
constexpr int kTcGroups = kTcEpiWarps / 4;  // column groups of a tile
constexpr int kTcGC = kTcCols / kTcGroups;  // columns of one group
constexpr int kTcThreads = (kTcEpiWarps + 2) * 32;  // + a producer warp and an MMA warp
static_assert(kTcGC % 32 == 0, "whole 32-column TMEM loads per group");
constexpr uint32_t kTcTmemCols = 256;  // potential pass: two accumulators of kTcCols columns
constexpr uint32_t kTcApplyTmemCols = 512;  // apply pass: two score accumulators + the result
// Weights p <= 1 of the apply passes are stored as fp16(2^15 p): the largest lands below
// fp16's maximum and weights down to 2^-39 keep their leading bits.
constexpr float kPScale = 32768.0f;
constexpr uint32_t kCoreLBO = 16u * 128u;  // next K-block of a core-matrix tile
constexpr uint32_t kCoreSBO = 128u;        // next 8-point group
// Dynamic shared memory a tensor-core pass may take (the opt-in limit is 227 KB; the
// kernels' static shared memory is at most 5 KB).
constexpr size_t kTcSmemBudget = 222u * 1024u;

template <int D>
struct TcShape {
  static constexpr int K = 2 * D;                  // [hi | lo] elements per point
  static constexpr int KSTEPS = D / 16;            // MMA K = 16 for fp16
  static constexpr uint32_t TILE_BYTES = 128u * K * 2u;
  static constexpr uint32_t LO_OFF = (D / 8) * kCoreLBO;  // first K-block of the lo half
  static constexpr uint32_t HY_BYTES = kTcCols * 4u;
  static constexpr uint32_t STAGE_BYTES = TILE_BYTES + 1024u;  // hy, padded to keep stages aligned
  static constexpr size_t SMEM = static_cast<size_t>(TILE_BYTES) + kTcStages * STAGE_BYTES;
};

// Byte offset of K element kk of point i in an operand image with K elements per point.
__host__ __device__ __forceinline__ int64_t tc_image_offset(int64_t i, int kk, int K) {
  const int64_t tile = i >> 7;
  const int r = static_cast<int>(i & 127);
  return tile * (128ll * K * 2) + (static_cast<int64_t>(kk >> 3) * 16 + (r >> 3)) * 128 +
         (r & 7) * 16 + (kk & 7) * 2;
}

// Shared-memory matrix descriptor: no swizzle, sm_100 version field. For K-major operands
// lbo steps along K and sbo along M/N; for MN-major operands lbo steps along K (the next 8
// rows of K) and sbo along M/N (the next 8 elements).
__device__ __forceinline__ uint64_t tc_smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Instruction descriptor of kind::f16: fp16 A and B, fp32 accumulate, M x N; A K-major,
// B K-major (b_mn = false) or MN-major (b_mn = true).
__host__ __device__ constexpr uint32_t tc_instr_desc(int M, int N, bool b_mn = false) {
  return (1u << 4) | (b_mn ? (1u << 16) : 0u) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
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

// The score tile of one 128-row block against one 128-key tile: three MMAs per 16-wide
// K-step (hi.hi, lo.hi, hi.lo) into the accumulator at tmem_d. a0 and b0 are the
// shared-memory addresses of the row and key images ([hi | lo], K-major).
// With accumulate set, the first MMA adds to the accumulator too (a later K-chunk of one
// score tile).
template <int D>
__device__ __forceinline__ void tc_issue_scores(uint32_t tmem_d, uint32_t a0, uint32_t b0,
                                                uint32_t idesc, bool accumulate = false) {
  using S = TcShape<D>;
#pragma unroll
  for (int s = 0; s < S::KSTEPS; ++s) {
    const uint32_t o = static_cast<uint32_t>(s) * 2u * kCoreLBO;
    tc_mma_f16(tmem_d, tc_smem_desc(a0 + o, kCoreLBO, kCoreSBO),
               tc_smem_desc(b0 + o, kCoreLBO, kCoreSBO), idesc,
               (s > 0 || accumulate) ? 1u : 0u);
    tc_mma_f16(tmem_d, tc_smem_desc(a0 + S::LO_OFF + o, kCoreLBO, kCoreSBO),
               tc_smem_desc(b0 + o, kCoreLBO, kCoreSBO), idesc, 1u);
    tc_mma_f16(tmem_d, tc_smem_desc(a0 + o, kCoreLBO, kCoreSBO),
               tc_smem_desc(b0 + S::LO_OFF + o, kCoreLBO, kCoreSBO), idesc, 1u);
  }
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

// 8 consecutive fp32 columns of this thread's TMEM lane; the caller waits.
__device__ __forceinline__ void tc_ld8_nowait(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
}

__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct TcParams {
  const unsigned char* row_img;  // query cloud's image, tiles of 128 points
  const unsigned char* key_img;  // streamed cloud's image
  const float* key_hy;           // hy of the streamed cloud, padded to whole tiles
  const float* row_nrm;          // |x_i|^2 of the query cloud (centred)
  int64_t key_tiles;             // tiles of 128 keys
  int64_t tiles_per_split;
  float c2;                      // 2 kappa / s^2: scale of the MMA result
  int32_t kc;                    // wide images (d > 64): 64-coordinate chunks per point
};

// Waits for phase `parity` of `bar`, giving up after kWaitLimitNs or as soon as another
// role of the CTA has raised `abort`. Between checks the thread sleeps in the barrier wait
// (up to 2 us per try), and the abort flag and the clock are read only every 16th try, so
// waiting warps leave the shared-memory and special-function issue queues to the warps
// that are computing.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t k = 1;; ++k) {
    if (mbar_try_wait_sleep(bar, parity, 2000u)) return true;
    if ((k & 15u) == 0u) {
      if (*abort) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---- epilogue pieces shared by the tensor-core kernels ------------------------------------

// Column pairs per pair whose exponentials the LSE epilogue computes on the FMA pipe
// (0: all on the MUFU unit).
constexpr int kTcPolyEvery = 4;

// Online max/sum of one row (its column group) over the score tiles: running offset m
// (log2 units, -inf until a real column sets it), base (m, or 0 before), mo = kappa |x|^2 + m
// subtracted from each score, and the running sums L (two lanes).
struct TcRowLse {
  float m, base, mo, knrm;
  u64 L;
};

__device__ __forceinline__ TcRowLse tc_row_lse_init(float knrm) {
  TcRowLse s;
  s.m = -INFINITY;
  s.base = 0.0f;
  s.mo = knrm;
  s.knrm = knrm;
  s.L = pk(0.0f, 0.0f);
  return s;
}

// Folds one tile into the row state: v holds the group's kTcGC raw scores (the MMA result),
// hy the group's key biases (shared memory, 16-byte aligned), c2 the score scale.
__device__ __forceinline__ void tc_lse_tile(TcRowLse& s, const float* v, const float* hy,
                                            u64 c2) {
  constexpr int GP = kTcGC / 2;  // column pairs of a group
  const ulonglong2* hv = reinterpret_cast<const ulonglong2*>(hy);
  u64 tv[GP];
  const u64 nmo = pk(-s.mo, -s.mo);
#pragma unroll
  for (int j = 0; j < GP; j += 2) {
    const ulonglong2 h = hv[j / 2];  // four biases in one 16-byte (broadcast) load
    tv[j] = add2(fma2(c2, pk(v[2 * j], v[2 * j + 1]), h.x), nmo);
    tv[j + 1] = add2(fma2(c2, pk(v[2 * j + 2], v[2 * j + 3]), h.y), nmo);
  }
  // the tile's maximum and, below, its sum as two interleaved chains (even and odd column
  // pairs): half the dependency depth for a thread that owns one row
  float a0, a1, b0, b1;
  upk(tv[0], a0, a1);
  upk(tv[1], b0, b1);
  float mxe = fmaxf(a0, a1), mxo = fmaxf(b0, b1);
#pragma unroll
  for (int j = 2; j < GP; j += 2) {
    upk(tv[j], a0, a1);
    mxe = max3(mxe, a0, a1);
    upk(tv[j + 1], b0, b1);
    mxo = max3(mxo, b0, b1);
  }
  const float mx = fmaxf(mxe, mxo);
  const float mx_abs = mx + s.base;
  if (mx_abs > s.m + kLazyThr && mx > kEmptyCut) {
    const float sc = ex2(s.m - mx_abs);
    s.L = mul2(s.L, pk(sc, sc));
    const u64 sh = pk(-mx, -mx);
#pragma unroll
    for (int j = 0; j < GP; ++j) tv[j] = add2(tv[j], sh);
    s.m = mx_abs;
    s.base = mx_abs;
    s.mo = s.knrm + s.m;
  }
  // One column pair in kTcPolyEvery takes its exponentials on the FMA pipe (ex2_poly2), the
  // rest on the MUFU unit, which is this pass's bound while issue slots are free.
  u64 se = pk(0.0f, 0.0f), so = pk(0.0f, 0.0f);
#pragma unroll
  for (int j = 0; j < GP; ++j) {
    u64 e;
    if (kTcPolyEvery > 0 && j % kTcPolyEvery == kTcPolyEvery - 1) {
      e = ex2_poly2(tv[j]);
    } else {
      float t0, t1;
      upk(tv[j], t0, t1);
      e = pk(ex2(t0), ex2(t1));
    }
    if (j & 1)
      so = add2(so, e);
    else
      se = add2(se, e);
  }
  s.L = add2(s.L, add2(se, so));
}

// Merges the column groups' states of every row and completes the row: the pass kind's
// finish (split mode: the row's partial). Called by every thread of the CTA once all roles
// are done; `merge` is shared scratch of kTcGroups x kTcRows entries.
template <int D>
__device__ __forceinline__ void tc_lse_finish(const PassParams& P, float2 (*merge)[kTcRows],
                                              const TcRowLse& s, bool epi, int grp, int r,
                                              int64_t i, int split) {
  float l0, l1;
  upk(s.L, l0, l1);
  if (epi) merge[grp][r] = make_float2(s.m, l0 + l1);
  __syncthreads();
  double dev = 0.0, mass = 0.0;
  if (epi && grp == 0 && i < P.n_rows) {
    float mm = -INFINITY;
#pragma unroll
    for (int q = 0; q < kTcGroups; ++q) mm = fmaxf(mm, merge[q][r].x);
    float l = 0.0f;
#pragma unroll
    for (int q = 0; q < kTcGroups; ++q) {
      const float2 o = merge[q][r];
      if (o.x != -INFINITY) l += o.y * ex2(o.x - mm);
    }
    if (P.n_splits == 1) {
      const double lse2 = static_cast<double>(mm) + log2(static_cast<double>(l));
      if (P.kind == kPot) {
        finish_pot<D>(P, i, lse2);
      } else if (P.kind == kLse) {
        P.lse_out[i] = static_cast<float>(lse2);
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

// The weights of one tile for the apply passes: q = 2^15 2^(score - offset) rounded to fp16,
// as packed pairs h2; L sums the rounded values.
__device__ __forceinline__ void tc_weights_tile(const float* v, const float* hy, u64 c2, u64 noff,
                                                u64& L, uint32_t* h2) {
  constexpr int GP = kTcGC / 2;
#pragma unroll
  for (int j = 0; j < GP; ++j) {
    float t0, t1;
    const ulonglong2 h4 = reinterpret_cast<const ulonglong2*>(hy)[j / 2];
    upk(add2(fma2(c2, pk(v[2 * j], v[2 * j + 1]), (j & 1) ? h4.y : h4.x), noff), t0, t1);
    const __half2 h = __floats2half2_rn(ex2(t0) * kPScale, ex2(t1) * kPScale);
    const float2 back = __half22float2(h);
    L = add2(L, pk(back.x, back.y));
    h2[j] = *reinterpret_cast<const uint32_t*>(&h);
  }
}

// Stores this thread's kTcGC weights (row r, column group grp) into a K-major weight tile:
// core(row group, key block) at (kb * 16 + r / 8) * 128 + (r % 8) * 16.
__device__ __forceinline__ void tc_store_weights(unsigned char* tile, int r, int grp,
                                                 const uint32_t* h2) {
  unsigned char* pt = tile + (r >> 3) * 128 + (r & 7) * 16;
#pragma unroll
  for (int c = 0; c < kTcGC / 8; ++c) {
    const int kb = grp * (kTcGC / 8) + c;
    *reinterpret_cast<uint4*>(pt + kb * 16 * 128) =
        make_uint4(h2[4 * c], h2[4 * c + 1], h2[4 * c + 2], h2[4 * c + 3]);
  }
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
  __shared__ float2 merge[kTcGroups][kTcRows];

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

  const int quarter = warp & 3, grp = warp >> 2;
  const int r = quarter * 32 + lane;
  const int64_t i = row0 + r;
  TcRowLse rs = tc_row_lse_init((i < P.n_rows) ? P.kappa_f * T.row_nrm[i] : 0.0f);

  if (warp == kTcEpiWarps) {
    // ---- producer: the row block once, then key tiles through the stage ring ----------
    if (lane == 0) {
      int issued = 0;
      mbar_expect_tx(&a_bar, S::TILE_BYTES);
      bulk_g2s(sA, T.row_img + (row0 >> 7) * S::TILE_BYTES, S::TILE_BYTES, &a_bar);
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % kTcStages;
        if (t >= kTcStages &&
            !tc_wait(&free_bar[st], static_cast<uint32_t>((t - kTcStages) / kTcStages) & 1u, abort))
          break;
        unsigned char* dst = sStage + st * S::STAGE_BYTES;
        const int64_t kt = t_begin + t;
        fence_proxy_async_smem();
        mbar_expect_tx(&full_bar[st], S::TILE_BYTES + S::HY_BYTES);
        bulk_g2s(dst, T.key_img + kt * S::TILE_BYTES, S::TILE_BYTES, &full_bar[st]);
        bulk_g2s(dst + S::TILE_BYTES, T.key_hy + kt * kTcCols, S::HY_BYTES, &full_bar[st]);
        ++issued;
      }
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
        tc_issue_scores<D>(tmem + static_cast<uint32_t>(b) * kTcCols, smem_u32(sA),
                           smem_u32(sStage + st * S::STAGE_BYTES), idesc);
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
    // ---- epilogue warps: online max/sum of one row over one column group of every tile --
    const u64 c2 = pk(T.c2, T.c2);
    for (int u = 0; u < n_tiles; ++u) {
      const int b = u & 1, st = u % kTcStages;
      if (!tc_wait(&mma_bar[b], static_cast<uint32_t>(u >> 1) & 1u, abort)) break;
      tc_fence_after();
      const float* hy = reinterpret_cast<const float*>(sStage + st * S::STAGE_BYTES + S::TILE_BYTES);
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(b) * kTcCols + grp * kTcGC;
      float v[kTcGC];
#pragma unroll
      for (int c = 0; c < kTcGC; c += 32) tc_ld32_nowait(tbase + c, v + c);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free_bar[b]);
      tc_lse_tile(rs, v, hy + grp * kTcGC, c2);
      // the stage is released once its biases have been read
      __syncwarp();
      if (lane == 0) mbar_arrive(&free_bar[st]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (abort_sh) {
    if (tid == 0) atomicOr(P.err, kErrTimeout);
  } else {
    tc_lse_finish<D>(P, merge, rs, warp < kTcEpiWarps, grp, r, i, split);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTcTmemCols));
}

// ---- the apply pass: sum_j p_ij U_j at fixed row offsets ------------------------------------

//   kApplyGrad: U = the key coordinates, q = p; out = the gradient 2 w_i (x_i - T_i).
//   kApplyPay:  U = a payload image (kPayChannels channels), q = p; out = mass_i sum q U / sum p.
//   kApplyDiff: U = the key coordinates, q = p (dg_j + (y_j - x_i).v_i) with a second score
//               W = V Y^T on the tensor cores; out = mass_i sum_j q_ij (y_j - x_i) / sum_j p_ij
//               (the difference pass of the Hessian-vector product).
enum TcApplyMode : int { kApplyGrad = 0, kApplyPay = 1, kApplyDiff = 2 };
constexpr int kPayChannels = 16;  // payload channels of one transport apply pass

struct TcApply {
  const float* row_lse;          // LSE2 of every query row (the offset), padding rows unread
  const float* row_mass;         // kApplyPay: plan mass of each row, or NULL (the row weight)
  const unsigned char* pay_img;  // kApplyPay: payload image, tiles of 128 keys x [hi | lo]
  const float* pay_inv_scale;    // kApplyPay: device scalar 1 / s_u of the payload image
  const float* x;                // kApplyGrad: query cloud (n_rows, d_real), caller order
  float* out;                    // results: row i, channel c at out[i * out_stride + c]
  int32_t out_k;                 // kApplyPay: channels written
  int32_t out_stride;
  float inv_key_scale;           // kApplyGrad, kApplyDiff: 1 / s of the key image
  double ctr[64];                // kApplyGrad, kApplyDiff: the centre the images were built about
  // kApplyDiff: the rows' vectors v_i as an image ([hi | lo], scaled by s_v), per row
  // (qs_i, x'_i.v_i) with q stored as fp16(qs_i q), the keys' dg padded to whole tiles, and
  // the device scalar 1 / s_v (the second score is W / (s_v s))
  const unsigned char* v_img;
  const float* v_row;
  const float* key_dg;
  const float* v_inv_scale;
};

template <int D, int NC, int MODE>
struct TcApplyShape {
  using S = TcShape<D>;
  static constexpr uint32_t PAY_BYTES = MODE == kApplyPay ? 128u * 2u * NC * 2u : 0u;
  static constexpr uint32_t HY_OFF = S::TILE_BYTES + PAY_BYTES;
  static constexpr uint32_t DG_OFF = HY_OFF + S::HY_BYTES;  // kApplyDiff: the keys' dg
  static constexpr uint32_t STAGE_BYTES = HY_OFF + 1024u;
  static constexpr uint32_t P_BYTES = 128u * 128u * 2u;  // one fp16 weight tile
  // the row image (and for kApplyDiff the rows' vector image) and two weight tiles
  static constexpr size_t BASE =
      static_cast<size_t>(S::TILE_BYTES) * (MODE == kApplyDiff ? 2u : 1u) + 2u * P_BYTES;
  // TMEM columns: two score accumulators, the second score (kApplyDiff), the result
  static constexpr uint32_t W_COL = 2u * kTcCols;
  static constexpr uint32_t O_COL = W_COL + (MODE == kApplyDiff ? kTcCols : 0u);
  static constexpr int STAGES = BASE + 3u * STAGE_BYTES <= kTcSmemBudget ? 3 : 2;
  static constexpr size_t SMEM = BASE + static_cast<size_t>(STAGES) * STAGE_BYTES;
  static constexpr uint32_t U_LO_OFF = (NC / 8) * kCoreLBO;  // lo half of the U operand
  static_assert(NC % 16 == 0 && NC >= 16 && NC <= 128, "MMA N of the result");
  static_assert(SMEM <= kTcSmemBudget, "shared memory");
  static_assert(O_COL + NC <= kTcApplyTmemCols, "tensor memory");
};

// Completes channel c of row i from its sums: a = sum_j q_ij U_jc and l = sum_j q_ij (the
// rounded, 2^15-scaled weights of the row).
template <int MODE>
__device__ __forceinline__ void tc_apply_finish(const PassParams& P, const TcApply& A, int64_t i,
                                                int c, double a, double l) {
  if constexpr (MODE == kApplyGrad) {
    if (c >= P.d_real) return;
    const double w = P.w ? static_cast<double>(P.w[i]) : static_cast<double>(P.w_uniform);
    const double t = A.ctr[c] + a / l;  // the barycentric projection T_i
    A.out[i * A.out_stride + c] =
        static_cast<float>(2.0 * w * (static_cast<double>(A.x[i * P.d_real + c]) - t));
  } else if constexpr (MODE == kApplyPay) {
    if (c >= A.out_k) return;
    const double mass = A.row_mass ? static_cast<double>(A.row_mass[i])
                                   : (P.w ? static_cast<double>(P.w[i])
                                          : static_cast<double>(P.w_uniform));
    A.out[i * A.out_stride + c] = static_cast<float>(l > 0.0 ? mass * a / l : 0.0);
  }
}

// kApplyDiff: channel c of row i from a = sum_j q'_ij y'_jc, lq = sum_j q'_ij (q' = qs_i q,
// fp16-rounded) and lp = sum_j p_ij: mass_i (a - x'_ic lq) / (qs_i lp).
__device__ __forceinline__ void tc_diff_finish(const PassParams& P, const TcApply& A, int64_t i,
                                               int c, double a, double lq, double lp) {
  if (c >= P.d_real) return;
  const double mass = A.row_mass ? static_cast<double>(A.row_mass[i])
                                 : (P.w ? static_cast<double>(P.w[i])
                                        : static_cast<double>(P.w_uniform));
  const double qs = static_cast<double>(A.v_row[2 * i]);
  const double xc = static_cast<double>(A.x[i * P.d_real + c]) - A.ctr[c];
  A.out[i * A.out_stride + c] =
      static_cast<float>(lp > 0.0 && qs > 0.0 ? mass * (a - xc * lq) / (qs * lp) : 0.0);
}

template <int D, int NC, int MODE>
__global__ void __launch_bounds__(kTcThreads, 1)
    lse_apply_tc_kernel(const PassParams P, const TcParams T, const TcApply A) {
  using S = TcShape<D>;
  using Sh = TcApplyShape<D, NC, MODE>;
  constexpr int ST = Sh::STAGES;
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint64_t full_bar[ST];   // tile landed
  __shared__ uint64_t free_bar[ST];   // stage reusable: result MMA commit + 8 epilogue warps
  __shared__ uint64_t mma_bar[2];     // score accumulator ready
  __shared__ uint64_t acc_free_bar[2];  // score accumulator read by the 8 epilogue warps
  __shared__ uint64_t p_full[2];      // weight tile written by the 8 epilogue warps
  __shared__ uint64_t p_free[2];      // weight tile read by its result MMAs
  __shared__ uint64_t w_free;         // kApplyDiff: second score read by the 8 epilogue warps
  __shared__ uint64_t a_bar, o_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float lsum[kTcGroups][kTcRows];   // per column group: sum of the rounded q'
  __shared__ float lpsum[kTcGroups][kTcRows];  // kApplyDiff: sum of the weights p

  constexpr bool DIFF = MODE == kApplyDiff;
  unsigned char* sA = smem;
  unsigned char* sV = smem + S::TILE_BYTES;  // kApplyDiff: the rows' vector image
  unsigned char* sP = smem + S::TILE_BYTES * (DIFF ? 2 : 1);
  unsigned char* sStage = sP + 2 * Sh::P_BYTES;
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
      mbar_init(&free_bar[s], kTcEpiWarps + 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&mma_bar[b], 1);
      mbar_init(&acc_free_bar[b], kTcEpiWarps);
      mbar_init(&p_full[b], kTcEpiWarps);
      mbar_init(&p_free[b], 1);
    }
    mbar_init(&w_free, kTcEpiWarps);
    mbar_init(&a_bar, 1);
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
  const uint32_t tmem_w = tmem + Sh::W_COL;  // kApplyDiff: the second score
  const uint32_t tmem_o = tmem + Sh::O_COL;  // the result accumulator, NC columns

  const int quarter = warp & 3, grp = warp >> 2;
  const int r = quarter * 32 + lane;
  const int64_t i = row0 + r;
  u64 L = pk(0.0f, 0.0f);   // epilogue: sum of this row's rounded weights q' over its group
  u64 Lp = pk(0.0f, 0.0f);  // kApplyDiff: sum of the weights p

  if (warp == kTcEpiWarps) {
    // ---- producer ---------------------------------------------------------------------
    if (lane == 0) {
      int issued = 0;
      mbar_expect_tx(&a_bar, S::TILE_BYTES * (DIFF ? 2u : 1u));
      bulk_g2s(sA, T.row_img + (row0 >> 7) * S::TILE_BYTES, S::TILE_BYTES, &a_bar);
      if constexpr (DIFF)
        bulk_g2s(sV, A.v_img + (row0 >> 7) * S::TILE_BYTES, S::TILE_BYTES, &a_bar);
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % ST;
        if (t >= ST && !tc_wait(&free_bar[st], static_cast<uint32_t>((t - ST) / ST) & 1u, abort))
          break;
        unsigned char* dst = sStage + st * Sh::STAGE_BYTES;
        const int64_t kt = t_begin + t;
        fence_proxy_async_smem();
        mbar_expect_tx(&full_bar[st], S::TILE_BYTES + Sh::PAY_BYTES + S::HY_BYTES *
                                                                     (DIFF ? 2u : 1u));
        bulk_g2s(dst, T.key_img + kt * S::TILE_BYTES, S::TILE_BYTES, &full_bar[st]);
        if constexpr (MODE == kApplyPay)
          bulk_g2s(dst + S::TILE_BYTES, A.pay_img + kt * Sh::PAY_BYTES, Sh::PAY_BYTES,
                   &full_bar[st]);
        bulk_g2s(dst + Sh::HY_OFF, T.key_hy + kt * kTcCols, S::HY_BYTES, &full_bar[st]);
        if constexpr (DIFF)
          bulk_g2s(dst + Sh::DG_OFF, A.key_dg + kt * kTcCols, S::HY_BYTES, &full_bar[st]);
        ++issued;
      }
      if (*abort) {
        (void)mbar_wait_bounded(&a_bar, 0);
        for (int t = (issued > ST ? issued - ST : 0); t < issued; ++t)
          (void)mbar_wait_bounded(&full_bar[t % ST], static_cast<uint32_t>(t / ST) & 1u);
      }
    }
  } else if (warp == kTcEpiWarps + 1) {
    // ---- MMA issuer: scores of tile t, then the result MMAs of tile t - 1 ---------------
    if (lane == 0) {
      const uint32_t idesc_s = tc_instr_desc(kTcRows, kTcCols);
      const uint32_t idesc_o = tc_instr_desc(kTcRows, NC, true);
      bool ok = tc_wait(&a_bar, 0, abort);
      for (int t = 0; ok && t <= n_tiles; ++t) {
        if (t < n_tiles) {
          const int st = t % ST, b = t & 1;
          if (!tc_wait(&full_bar[st], static_cast<uint32_t>(t / ST) & 1u, abort)) break;
          if (t >= 2 && !tc_wait(&acc_free_bar[b], static_cast<uint32_t>((t - 2) >> 1) & 1u, abort))
            break;
          tc_fence_after();
          tc_issue_scores<D>(tmem + static_cast<uint32_t>(b) * kTcCols, smem_u32(sA),
                             smem_u32(sStage + st * Sh::STAGE_BYTES), idesc_s);
          if constexpr (DIFF) {
            // the second score W = V Y^T, single-buffered: tile t - 1's must have been read
            if (t >= 1 && !tc_wait(&w_free, static_cast<uint32_t>(t - 1) & 1u, abort)) break;
            tc_fence_after();
            tc_issue_scores<D>(tmem_w, smem_u32(sV), smem_u32(sStage + st * Sh::STAGE_BYTES),
                               idesc_s);
          }
          tc_commit(&mma_bar[b]);
        }
        if (t >= 1) {
          const int u = t - 1, su = u % ST, pb = u & 1;
          if (!tc_wait(&p_full[pb], static_cast<uint32_t>(u >> 1) & 1u, abort)) break;
          tc_fence_after();
          const uint32_t pa = smem_u32(sP + pb * Sh::P_BYTES);
          const uint32_t ub = smem_u32(sStage + su * Sh::STAGE_BYTES) +
                              (MODE == kApplyPay ? S::TILE_BYTES : 0u);
          // U along N (coordinates or channels), keys along K: MN-major
#pragma unroll
          for (int s = 0; s < kTcCols / 16; ++s) {
            const uint64_t ad = tc_smem_desc(pa + s * 2u * kCoreLBO, kCoreLBO, kCoreSBO);
            const uint32_t ko = static_cast<uint32_t>(s) * 2u * kCoreSBO;  // next 16 keys
            tc_mma_f16(tmem_o, ad, tc_smem_desc(ub + ko, kCoreSBO, kCoreLBO), idesc_o,
                       (u > 0 || s > 0) ? 1u : 0u);
            tc_mma_f16(tmem_o, ad, tc_smem_desc(ub + Sh::U_LO_OFF + ko, kCoreSBO, kCoreLBO),
                       idesc_o, 1u);
          }
          tc_commit(&free_bar[su]);
          tc_commit(&p_free[pb]);
        }
      }
      // Every MMA this thread issued has completed once o_bar fires; wait for it here so
      // that TMEM is never released under a running MMA, whatever the other roles did.
      tc_commit(&o_bar);
      (void)mbar_wait_bounded(&o_bar, 0);
    }
  } else {
    // ---- epilogue warps: weights of one row over one column group of every tile ---------
    constexpr int GP = kTcGC / 2;  // column pairs of a group
    float off = 1.0e30f;  // padding rows: every weight is 0
    if (i < P.n_rows) off = P.kappa_f * T.row_nrm[i] + A.row_lse[i];
    const u64 c2 = pk(T.c2, T.c2);
    const u64 noff = pk(-off, -off);
    // kApplyDiff: q'_ij = qs_i p_ij (dg_j + w_scale W_ij - x'_i.v_i)
    float qs = 0.0f, xv = 0.0f;
    if (DIFF && i < P.n_rows) {
      qs = A.v_row[2 * i];
      xv = A.v_row[2 * i + 1];
    }
    const float w_scale = DIFF ? *A.v_inv_scale * A.inv_key_scale : 0.0f;
    const u64 wsc = pk(w_scale, w_scale);
    const u64 nxv = pk(-xv, -xv);
    for (int u = 0; u < n_tiles; ++u) {
      const int b = u & 1, st = u % ST, pb = u & 1;
      if (!tc_wait(&mma_bar[b], static_cast<uint32_t>(u >> 1) & 1u, abort)) break;
      tc_fence_after();
      const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t tbase = tmem + lane_off + static_cast<uint32_t>(b) * kTcCols + grp * kTcGC;
      const u64* hv = reinterpret_cast<const u64*>(sStage + st * Sh::STAGE_BYTES + Sh::HY_OFF) +
                      grp * GP;
      uint32_t h2[GP];  // fp16 pairs of the weights q' (2^15 p unless kApplyDiff)
      if constexpr (!DIFF) {
        float v[kTcGC];
#pragma unroll
        for (int c = 0; c < kTcGC; c += 32) tc_ld32_nowait(tbase + c, v + c);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_free_bar[b]);
        tc_weights_tile(v, reinterpret_cast<const float*>(hv), c2, noff, L, h2);
      } else {
        const u64* dv = reinterpret_cast<const u64*>(sStage + st * Sh::STAGE_BYTES + Sh::DG_OFF) +
                        grp * GP;
        const uint32_t wbase = tmem_w + lane_off + grp * kTcGC;
        constexpr int NCH = kTcGC / 32;
#pragma unroll
        for (int h = 0; h < NCH; ++h) {  // chunks of 32 columns
          float v[32], wv[32];
          tc_ld32_nowait(tbase + 32 * h, v);
          tc_ld32_nowait(wbase + 32 * h, wv);
          tc_wait_ld();
          if (h == NCH - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&acc_free_bar[b]);
              mbar_arrive(&w_free);
            }
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int jj = 16 * h + j;
            float t0, t1, p0, p1, f0, f1;
            upk(add2(fma2(c2, pk(v[2 * j], v[2 * j + 1]), hv[jj]), noff), t0, t1);
            p0 = ex2(t0);
            p1 = ex2(t1);
            Lp = add2(Lp, pk(p0, p1));
            upk(add2(fma2(wsc, pk(wv[2 * j], wv[2 * j + 1]), dv[jj]), nxv), f0, f1);
            const __half2 hq = __floats2half2_rn(qs * p0 * f0, qs * p1 * f1);
            const float2 back = __half22float2(hq);
            L = add2(L, pk(back.x, back.y));
            h2[jj] = *reinterpret_cast<const uint32_t*>(&hq);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&free_bar[st]);  // its hy has been read
      if (u >= 2 && !tc_wait(&p_free[pb], static_cast<uint32_t>((u - 2) >> 1) & 1u, abort)) break;
      tc_store_weights(sP + pb * Sh::P_BYTES, r, grp, h2);
      fence_proxy_async_smem();  // the generic-proxy writes, before the MMA reads them
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[pb]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  {
    float l0, l1, p0, p1;
    upk(L, l0, l1);
    upk(Lp, p0, p1);
    if (warp < kTcEpiWarps) {
      lsum[grp][r] = l0 + l1;
      lpsum[grp][r] = p0 + p1;
    }
  }
  __syncthreads();
  if (abort_sh) {
    if (tid == 0) atomicOr(P.err, kErrTimeout);
  } else if (warp < 8) {
    // The result accumulator: this warp's rows, channels [half * NC / 2, (half + 1) * NC / 2)
    // (the warps of the first two column groups).
    const int half = grp;
    if (mbar_wait_bounded(&o_bar, 0)) {
      tc_fence_after();
      constexpr int NH = NC / 2;
      float o[NH];
      const uint32_t obase = tmem_o + (static_cast<uint32_t>(quarter * 32) << 16) + half * NH;
#pragma unroll
      for (int c = 0; c < NH; c += 8) tc_ld8_nowait(obase + c, o + c);
      tc_wait_ld();
      double l = 0.0, lp = 0.0;
#pragma unroll
      for (int q = 0; q < kTcGroups; ++q) {
        l += static_cast<double>(lsum[q][r]);
        lp += static_cast<double>(lpsum[q][r]);
      }
      const double inv = MODE == kApplyPay ? static_cast<double>(*A.pay_inv_scale)
                                           : static_cast<double>(A.inv_key_scale);
      if (i < P.n_rows) {
        if (P.n_splits == 1) {
#pragma unroll
          for (int c = 0; c < NH; ++c) {
            const double a = static_cast<double>(o[c]) * inv;
            if constexpr (DIFF)
              tc_diff_finish(P, A, i, half * NH + c, a, l, lp);
            else
              tc_apply_finish<MODE>(P, A, i, half * NH + c, a, l);
          }
        } else {
          // partials: [sum q'][channels][sum p (kApplyDiff)], split-major
          constexpr int NP = NC + (DIFF ? 1 : 0);
          const int64_t ps = static_cast<int64_t>(split);
          if (half == 0) P.part_l[ps * P.rows_pad + i] = static_cast<float>(l);
          if (DIFF && half == 0) P.part_a[(ps * NP + NC) * P.rows_pad + i] = static_cast<float>(lp);
#pragma unroll
          for (int c = 0; c < NH; ++c)
            P.part_a[(ps * NP + half * NH + c) * P.rows_pad + i] =
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

// Sums the column splits' partials of an apply pass (the offsets are fixed, so partials
// add) and completes each row.
template <int NC, int MODE>
__global__ void __launch_bounds__(256) tc_apply_combine_kernel(const PassParams P, const TcApply A) {
  constexpr bool DIFF = MODE == kApplyDiff;
  constexpr int NP = NC + (DIFF ? 1 : 0);
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= P.n_rows) return;
  double l = 0.0, lp = 0.0;
  for (int s = 0; s < P.n_splits; ++s) {
    l += P.part_l[static_cast<int64_t>(s) * P.rows_pad + i];
    if (DIFF) lp += P.part_a[(static_cast<int64_t>(s) * NP + NC) * P.rows_pad + i];
  }
  for (int c = 0; c < NC; ++c) {
    double a = 0.0;
    for (int s = 0; s < P.n_splits; ++s)
      a += P.part_a[(static_cast<int64_t>(s) * NP + c) * P.rows_pad + i];
    if constexpr (DIFF)
      tc_diff_finish(P, A, i, c, a, l, lp);
    else
      tc_apply_finish<MODE>(P, A, i, c, a, l);
  }
}

// ---- preparation for the tensor-core passes -----------------------------------------------

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

// The operand image of one cloud ([hi | lo] of the centred, scaled coordinates) and its
// centred squared norms, for all padded points.
template <int D>
__global__ void __launch_bounds__(256) build_image_kernel(const float* pts, int64_t count,
                                                          int32_t d_real, const TcCenter ctr,
                                                          float scale, unsigned char* img,
                                                          float* nrm, int64_t count_pad) {
  constexpr int K = 2 * D;
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
    *reinterpret_cast<__half*>(img + tc_image_offset(i, k, K)) = hi;
    *reinterpret_cast<__half*>(img + tc_image_offset(i, D + k, K)) = lo;
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

// Largest |u| over channels [0, k) of a row-major (count, stride) array, as float bits.
__global__ void __launch_bounds__(256) pay_maxabs_kernel(const float* u, int64_t count, int k,
                                                         int stride, unsigned* maxabs_bits) {
  float mx = 0.0f;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < count * k;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x)
    mx = fmaxf(mx, fabsf(u[(t / k) * stride + t % k]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) atomicMax(maxabs_bits, __float_as_uint(mx));
}

// Payload image of a transport apply pass: channels [0, k) of u scaled by the power of two
// s = 2^floor(log2(16384 / max|u|)) and split into [hi | lo] fp16 (NC channels per point,
// padding channels and points zero), in the core-matrix layout of the key images. Thread 0
// of block 0 also stores 1 / s.
template <int NC>
__global__ void __launch_bounds__(256) build_pay_image_kernel(const float* u, int64_t count,
                                                              int64_t count_pad, int k,
                                                              int stride,
                                                              const unsigned* maxabs_bits,
                                                              unsigned char* img,
                                                              float* inv_scale) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const float mx = __uint_as_float(*maxabs_bits);
  int e = 0;
  if (mx > 0.0f) e = static_cast<int>(floorf(log2f(16384.0f / mx)));
  e = max(-120, min(120, e));
  const float scale = exp2f(static_cast<float>(e));
  if (i == 0) *inv_scale = exp2f(static_cast<float>(-e));
  if (i >= count_pad) return;
#pragma unroll 4
  for (int c = 0; c < NC; ++c) {
    const float v = (i < count && c < k) ? u[i * stride + c] * scale : 0.0f;
    const __half hi = __float2half_rn(v);
    const __half lo = __float2half_rn(v - __half2float(hi));
    *reinterpret_cast<__half*>(img + tc_image_offset(i, c, 2 * NC)) = hi;
    *reinterpret_cast<__half*>(img + tc_image_offset(i, NC + c, 2 * NC)) = lo;
  }
}

// The difference pass's key column dg, zero-padded to whole tiles, and max |dg| (float bits).
__global__ void __launch_bounds__(256) dg_prep_kernel(const float* dg, int64_t count,
                                                      int64_t count_pad, float* dg_pad,
                                                      unsigned* maxabs_bits) {
  float mx = 0.0f;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < count_pad;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = j < count ? dg[j] : 0.0f;
    dg_pad[j] = v;
    mx = fmaxf(mx, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) atomicMax(maxabs_bits, __float_as_uint(mx));
}

// The difference pass's row side: the image of the vectors v_i (scaled by the power of two
// s_v = 2^floor(log2(16384 / max|v|)), [hi | lo]), 1 / s_v, and per row
//   qs_i = 2^14 / (max|dg| + |v_i| (r_key + |x'_i|))   and   x'_i.v_i,
// where |dg_j + (y'_j - x'_i).v_i| <= max|dg| + |v_i| (|y'_j| + |x'_i|) and r_key bounds
// |y'_j|, so |qs_i p_ij (dg_j + (y'_j - x'_i).v_i)| <= 2^14 for p <= 1 (fp16 range).
template <int D>
__global__ void __launch_bounds__(256) build_vrow_image_kernel(
    const float* v, const float* x, int64_t count, int64_t count_pad, int32_t d_real,
    const TcCenter ctr, const unsigned* vmax_bits, const unsigned* dgmax_bits, float r_key,
    unsigned char* img, float* v_row, float* inv_scale) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const float mx = __uint_as_float(*vmax_bits);
  int e = 0;
  if (mx > 0.0f) e = static_cast<int>(floorf(log2f(16384.0f / mx)));
  e = max(-120, min(120, e));
  const float scale = exp2f(static_cast<float>(e));
  if (i == 0) *inv_scale = exp2f(static_cast<float>(-e));
  if (i >= count_pad) return;
  double vv = 0.0, xx = 0.0, xv = 0.0;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    float u = 0.0f;
    if (i < count && k < d_real) {
      const double vk = static_cast<double>(v[i * d_real + k]);
      const double xk = static_cast<double>(x[i * d_real + k]) - ctr.c[k];
      vv += vk * vk;
      xx += xk * xk;
      xv += xk * vk;
      u = static_cast<float>(vk * scale);
    }
    const __half hi = __float2half_rn(u);
    const __half lo = __float2half_rn(u - __half2float(hi));
    *reinterpret_cast<__half*>(img + tc_image_offset(i, k, 2 * D)) = hi;
    *reinterpret_cast<__half*>(img + tc_image_offset(i, D + k, 2 * D)) = lo;
  }
  const double bound = static_cast<double>(__uint_as_float(*dgmax_bits)) +
                       sqrt(vv) * (static_cast<double>(r_key) + sqrt(xx));
  v_row[2 * i] = i < count && bound > 0.0 ? static_cast<float>(16384.0 / bound) : 0.0f;
  v_row[2 * i + 1] = static_cast<float>(xv);
}

}  // namespace fs
