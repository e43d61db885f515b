// fs_small.cuh -- small problems solved in one launch on a thread-block cluster (sm_100a).
//
// A fixed-count alternating solve (SinkSLOT README, API Reference: variant "alternating",
// stop_mode "fixed") of a problem with a few million pairs costs a few microseconds of
// exponentials per half-iteration, less than the launches, drains and merges of the
// streaming passes around it. Here one cluster of up to 16 CTAs runs every iteration in a
// single kernel. Every CTA stages both clouds (coordinate-major) with their log2 weights in
// shared memory once, and keeps the biases H_j = kappa pot_j + log2 w_j of both clouds there
// too. Each half-iteration the rows go in groups of 32, one row per lane, the groups dealt to
// the CTAs in turn; a CTA gives each of its groups 32 / WG warps (WG groups at a time), one
// slice of the keys per warp, read by all its lanes at once (two keys per packed fp32x2
// operation, the running max / sum of the lane's row kept lazily). The slices' (max, sum)
// pairs meet in shared memory, the group's first warp merges them, writes each row's new
// potential to global memory and its new bias into the bias array of EVERY CTA of the
// cluster (distributed shared memory stores), which the next half-iteration reads as its
// key biases. A hardware cluster barrier (release / acquire at cluster scope) ends each
// half-iteration. It cannot wait forever: every CTA of the cluster runs the same number of
// half-iterations and no CTA leaves early.
//
// The score is the direct difference z_ij = H_j - kappa |x_i - y_j|^2 in fp32 (the most
// accurate form; the oracle's is the same in fp64), the log-sum-exp online in base 2.
#pragma once

#include "fs_kernels.cuh"

namespace fs {

constexpr int kSmallThreads = 1024;  // 8 warps per scheduler to hide shared-memory latency
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallMaxCluster = 16;                   // CTAs (SMs); a non-portable size
constexpr int64_t kSmallMaxPairs = int64_t(1) << 22;   // n * m at most
constexpr size_t kSmallSmemBudget = 200u * 1024u;      // a CTA's shared memory at most

// Points per cloud as staged: padded to a multiple of 512, so that each of up to 32 key
// slices holds whole groups of kSmallGroup key pairs (padding keys carry log2(0) and add
// nothing).
constexpr int kSmallGroup = 8;  // key pairs per step (16 independent exponentials per lane)
__host__ __device__ constexpr int64_t small_pad(int64_t count) {
  return (count + 511) / 512 * 512;
}

struct SmallParams {
  const float* x;       // (n, d) caller order
  const float* y;       // (m, d)
  const float* a;       // (n,) or NULL: uniform wa
  const float* b;       // (m,) or NULL: uniform wb
  float wa, wb;
  const float* g_init;  // (m,) or NULL: g = 0
  float* f;             // (n,) output and iterate
  float* g;             // (m,) output and iterate (may alias g_init)
  int32_t n, m;
  int32_t d;            // true dimension (<= D)
  int32_t n_iters;
  double kappa;         // log2(e) / eps
  double inv_kappa;     // eps ln 2
  unsigned* err;        // the workspace error word (a wait that timed out sets kErrTimeout)
};

__device__ __forceinline__ void cluster_barrier() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ unsigned cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ unsigned cluster_size() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// Shared memory of one CTA: both clouds coordinate-major (D coordinate arrays and the log2
// weights, padded counts), the biases of both clouds, and the warps' per-row partials.
__host__ __device__ inline size_t small_smem_bytes(int64_t n, int64_t m, int D) {
  const int64_t np = small_pad(n), mp = small_pad(m);
  return static_cast<size_t>((np + mp) * (D + 2) + 2 * kSmallWarps * 32) * sizeof(float);
}

// Stores v at the address of `local` in the shared memory of CTA `rank` of the cluster and
// counts its 4 bytes on that CTA's mbarrier at the address of `bar` (asynchronous store).
__device__ __forceinline__ void st_async_cluster(float* local, unsigned rank, float v,
                                                 uint64_t* bar) {
  uint32_t ra, rb;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)),
               "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(smem_u32(bar)),
               "r"(rank));
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(
                   ra),
               "r"(__float_as_uint(v)), "r"(rb)
               : "memory");
}

// Bounded wait for a phase of an mbarrier that other CTAs of the cluster complete, with
// acquire semantics at cluster scope (their stores are then visible here).
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (true) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000u)
        : "memory");
    if (done) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// The bias of a point from its (float) potential and log2 weight, in double, rounded once.
__device__ __forceinline__ float small_bias(double kappa, float pot, float lw) {
  return lw > kLogZero ? static_cast<float>(kappa * static_cast<double>(pot) +
                                            static_cast<double>(lw))
                       : kLogZero;
}

template <int D>
__global__ void __launch_bounds__(kSmallThreads) small_solve_kernel(const SmallParams S) {
  extern __shared__ __align__(16) float sm[];
  const int np = static_cast<int>(small_pad(S.n)), mp = static_cast<int>(small_pad(S.m));
  float* sx = sm;                       // x: [D][np] coordinates, then [np] log2 a
  float* sy = sx + (D + 1) * np;        // y: [D][mp], then [mp] log2 b
  float* hx = sy + (D + 1) * mp;        // biases of x (the keys of the g-updates)
  float* hy = hx + np;                  // biases of y (the keys of the f-updates)
  auto part = reinterpret_cast<float(*)[kSmallWarps][32]>(hy + mp);  // [max | sum][warp][lane]
  // one per parity of the half-iteration: completes when every row's new bias of that
  // half-iteration has landed in this CTA's shared memory
  __shared__ uint64_t hbar[2];
  const unsigned crank = cluster_rank(), csize = cluster_size();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // both clouds once, with their log2 weights (kLogZero for a zero weight and for padding)
  for (int t = tid; t < np + mp; t += kSmallThreads) {
    const bool is_x = t < np;
    const int j = is_x ? t : t - np;
    const int count = is_x ? S.n : S.m, pad = is_x ? np : mp;
    const float* src = is_x ? S.x : S.y;
    float* dst = is_x ? sx : sy;
#pragma unroll
    for (int k = 0; k < D; ++k)
      dst[k * pad + j] = (j < count && k < S.d) ? src[static_cast<int64_t>(j) * S.d + k] : 0.0f;
    float lw = kLogZero;
    if (j < count) {
      const float w = is_x ? (S.a ? S.a[j] : S.wa) : (S.b ? S.b[j] : S.wb);
      if (w > 0.0f) lw = static_cast<float>(log2(static_cast<double>(w)));
    }
    dst[D * pad + j] = lw;
    // the biases: y's from g_init (or 0); x's are written by the first f-update (padding
    // entries keep log2(0))
    if (is_x)
      hx[j] = kLogZero;
    else
      hy[j] = j < count ? small_bias(S.kappa, S.g_init ? S.g_init[j] : 0.0f, lw) : kLogZero;
  }
  if (tid == 0) {
    mbar_init(&hbar[0], 1);
    mbar_init(&hbar[1], 1);
    fence_mbar_init();
  }
  // every CTA's arrays and mbarriers initialised before any CTA stores into them
  cluster_barrier();
  const u64 nkap = pk(-static_cast<float>(S.kappa), -static_cast<float>(S.kappa));
  for (int h = 0; h < 2 * S.n_iters; ++h) {
    const bool rows_x = (h & 1) == 0;  // f-update first, then the g-update
    uint64_t* bar = &hbar[h & 1];
    if (tid == 0) mbar_expect_tx(bar, 4u * static_cast<uint32_t>(rows_x ? S.n : S.m));
    const float* R = rows_x ? sx : sy;
    const float* K = rows_x ? sy : sx;
    const int nr = rows_x ? S.n : S.m;
    const int rpad = rows_x ? np : mp, kpad = rows_x ? mp : np;
    float* potr = rows_x ? S.f : S.g;
    float* hr = rows_x ? hx : hy;  // where the rows' new biases go (in every CTA)
    const u64* kc[D];
#pragma unroll
    for (int k = 0; k < D; ++k) kc[k] = reinterpret_cast<const u64*>(K + k * kpad);
    const u64* hv = reinterpret_cast<const u64*>(rows_x ? hy : hx);
    // Rows in groups of 32 (lane l: row 32 g + l), groups dealt to the CTAs in turn; a CTA
    // takes WG of its groups at a time and gives each S = 32 / WG warps, one slice of the
    // keys each (kSmallGroup key pairs per step, read by all lanes at once). Each warp's
    // (max, sum) per row goes to shared memory, and the group's first warp merges the S
    // slices of its rows.
    const int ngroups = (nr + 31) / 32;
    const int gpc = (ngroups + static_cast<int>(csize) - 1) / static_cast<int>(csize);
    int wg = 1;
    while (wg < gpc && wg < kSmallWarps) wg *= 2;
    const int slices = kSmallWarps / wg;
    const int slot = warp / slices, slice = warp % slices;
    const int per = kpad / 2 / slices;  // key pairs per slice (kpad / 2 is a multiple of 256)
    const int q0 = slice * per;
    for (int round = 0; round * wg < gpc; ++round) {
      const int gl = round * wg + slot;
      const int group = static_cast<int>(crank) + gl * static_cast<int>(csize);
      const bool active = gl < gpc && group < ngroups;  // the same for the whole warp
      const int i = group * 32 + lane;
      float mr = -INFINITY;
      u64 sr = pk(0.0f, 0.0f);
      if (active) {
        const int ic = i < nr ? i : nr - 1;  // lanes past the last row repeat it
        u64 xi[D];
#pragma unroll
        for (int k = 0; k < D; ++k) {
          const float c = R[k * rpad + ic];
          xi[k] = pk(c, c);
        }
        for (int q = q0; q < q0 + per; q += kSmallGroup) {
          u64 z[kSmallGroup];
          float gm = -INFINITY;
#pragma unroll
          for (int t = 0; t < kSmallGroup; ++t) {
            u64 acc = pk(0.0f, 0.0f);
#pragma unroll
            for (int k = 0; k < D; ++k) {
              const u64 dk = sub2(xi[k], kc[k][q + t]);
              acc = fma2(dk, dk, acc);
            }
            z[t] = fma2(nkap, acc, hv[q + t]);
            float z0, z1;
            upk(z[t], z0, z1);
            gm = max3(gm, z0, z1);
          }
          if (gm > mr + kLazyThr && gm > kEmptyCut) {
            const float sc = mr == -INFINITY ? 0.0f : ex2(mr - gm);
            sr = mul2(sr, pk(sc, sc));
            mr = gm;
          }
          if (mr != -INFINITY) {
            const u64 nm = pk(-mr, -mr);
#pragma unroll
            for (int t = 0; t < kSmallGroup; ++t) {
              float z0, z1;
              upk(add2(z[t], nm), z0, z1);
              sr = add2(sr, pk(ex2(z0), ex2(z1)));
            }
          }
        }
      }
      float s0, s1;
      upk(sr, s0, s1);
      part[0][warp][lane] = mr;
      part[1][warp][lane] = s0 + s1;
      __syncthreads();
      if (active && slice == 0) {
        // the slices' largest offset, then their sums scaled to it: independent terms
        // instead of a chain of pairwise merges
        float m = -INFINITY, sum = 0.0f;
        for (int j = 0; j < slices; ++j) m = fmaxf(m, part[0][warp + j][lane]);
        if (m != -INFINITY) {
          for (int j = 0; j < slices; ++j) {
            const float mj = part[0][warp + j][lane];
            if (mj != -INFINITY) sum = fmaf(part[1][warp + j][lane], ex2(mj - m), sum);
          }
        }
        if (i < nr) {
          // log2 of the sum in fp32 (2^-23 relative on a value below ~25, ~3e-6 log2 units,
          // far below the potentials' fp32 rounding); the rest in double as the other passes
          const double lse2 = static_cast<double>(m) + static_cast<double>(log2f(sum));
          const float pot = static_cast<float>(-lse2 * S.inv_kappa);
          potr[i] = pot;
          const float hnew = small_bias(S.kappa, pot, R[D * rpad + i]);
          // the new bias into every CTA of the cluster
          for (unsigned c = 0; c < csize; ++c) st_async_cluster(hr + i, c, hnew, bar);
        }
      }
      __syncthreads();  // the partials are read before the next round writes them
    }
    // Every row's new bias of this half-iteration has reached this CTA: all CTAs have also
    // finished reading the key biases of this half-iteration (each CTA's stores follow its
    // last read of them), so the next one may overwrite them.
    const bool ok = mbar_wait_cluster_bounded(bar, static_cast<uint32_t>(h >> 1) & 1u);
    if (__syncthreads_or(!ok)) {
      if (tid == 0) atomicOr(S.err, kErrTimeout);
      break;
    }
  }
  // no CTA leaves while stores into its shared memory could still be in flight
  cluster_barrier();
}

}  // namespace fs
