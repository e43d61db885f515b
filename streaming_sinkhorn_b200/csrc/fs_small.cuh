// fs_small.cuh -- small problems solved in one launch on a thread-block cluster (sm_100a).
//
// A fixed-count alternating solve (SinkSLOT README, API Reference: variant "alternating",
// stop_mode "fixed") of a problem with a few million pairs costs a few microseconds of
// exponentials per half-iteration, less than the launches, drains and merges of the
// streaming passes around it. Here one cluster of up to 16 CTAs runs every iteration in a
// single kernel. Every CTA stages both clouds (coordinate-major) with their log2 weights in
// shared memory once, and keeps the biases H_j = kappa pot_j + log2 w_j of both clouds there
// too. Each half-iteration its warps take rows two at a time (the 32 lanes of a warp split
// the keys, each key pair loaded once for both rows, two keys per packed fp32x2 operation),
// merge their (max, sum) pairs by shuffles, write each row's new potential to global memory
// and its new bias into the bias array of EVERY CTA of the cluster (distributed shared
// memory stores), which the next half-iteration reads as its key biases. A hardware
// cluster barrier (release / acquire at cluster scope) ends each half-iteration. It cannot
// wait forever: every CTA of the cluster runs the same number of half-iterations and no CTA
// leaves early.
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
constexpr size_t kSmallSmemBudget = 200u * 1024u;      // both staged clouds at most

// Points per cloud as staged: padded to a multiple of 512 so that every lane takes whole
// groups of kSmallGroup key pairs (padding keys carry log2(0) and add nothing).
constexpr int kSmallGroup = 4;  // key pairs per lane per step and row (two rows: 16 exponentials)
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

// Merges the (max, sum) pair of another lane into this one; an empty pair has max -inf.
__device__ __forceinline__ void merge_max_sum(float& mx, float& s, float mo, float so) {
  const float M = fmaxf(mx, mo);
  if (M == -INFINITY) return;
  s = (mx == -INFINITY ? 0.0f : s * ex2(mx - M)) + (mo == -INFINITY ? 0.0f : so * ex2(mo - M));
  mx = M;
}

// Shared memory of one CTA: both clouds coordinate-major (D coordinate arrays and the log2
// weights, padded counts) and the biases of both clouds.
__host__ __device__ inline size_t small_smem_bytes(int64_t n, int64_t m, int D) {
  const int64_t np = small_pad(n), mp = small_pad(m);
  return static_cast<size_t>((np + mp) * (D + 2)) * sizeof(float);
}

// Stores v at the address of `local` in the shared memory of CTA `rank` of the cluster.
__device__ __forceinline__ void st_cluster(float* local, unsigned rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)),
               "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
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
  // every CTA's arrays initialised before any CTA stores into them
  cluster_barrier();
  const u64 nkap = pk(-static_cast<float>(S.kappa), -static_cast<float>(S.kappa));
  const int stride = static_cast<int>(csize) * kSmallWarps;  // warps of the cluster
  for (int h = 0; h < 2 * S.n_iters; ++h) {
    const bool rows_x = (h & 1) == 0;  // f-update first, then the g-update
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
    // rows i and i + stride of this warp at once; a lane takes key pairs lane + 32 t,
    // kSmallGroup at a time, and rescales a row's running sum only when a group's maximum
    // exceeds its offset by more than kLazyThr
    for (int i = static_cast<int>(crank) * kSmallWarps + warp; i < nr; i += 2 * stride) {
      const int i2 = i + stride < nr ? i + stride : i;  // a lone last row is computed twice
      u64 xa[D], xb[D];
#pragma unroll
      for (int k = 0; k < D; ++k) {
        const float ca = R[k * rpad + i], cb = R[k * rpad + i2];
        xa[k] = pk(ca, ca);
        xb[k] = pk(cb, cb);
      }
      float ma = -INFINITY, mb = -INFINITY;
      u64 sa = pk(0.0f, 0.0f), sb = pk(0.0f, 0.0f);
      for (int q0 = lane; q0 < kpad / 2; q0 += 32 * kSmallGroup) {
        u64 za[kSmallGroup], zb[kSmallGroup];
        float ga = -INFINITY, gb = -INFINITY;
#pragma unroll
        for (int t = 0; t < kSmallGroup; ++t) {
          const int q = q0 + 32 * t;
          u64 aa = pk(0.0f, 0.0f), ab = pk(0.0f, 0.0f);
#pragma unroll
          for (int k = 0; k < D; ++k) {
            const u64 yk = kc[k][q];
            const u64 da = sub2(xa[k], yk), db = sub2(xb[k], yk);
            aa = fma2(da, da, aa);
            ab = fma2(db, db, ab);
          }
          const u64 hq = hv[q];
          za[t] = fma2(nkap, aa, hq);
          zb[t] = fma2(nkap, ab, hq);
          float z0, z1;
          upk(za[t], z0, z1);
          ga = max3(ga, z0, z1);
          upk(zb[t], z0, z1);
          gb = max3(gb, z0, z1);
        }
        if (ga > ma + kLazyThr && ga > kEmptyCut) {
          const float sc = ma == -INFINITY ? 0.0f : ex2(ma - ga);
          sa = mul2(sa, pk(sc, sc));
          ma = ga;
        }
        if (gb > mb + kLazyThr && gb > kEmptyCut) {
          const float sc = mb == -INFINITY ? 0.0f : ex2(mb - gb);
          sb = mul2(sb, pk(sc, sc));
          mb = gb;
        }
        if (ma != -INFINITY) {
#pragma unroll
          for (int t = 0; t < kSmallGroup; ++t) {
            float z0, z1;
            upk(za[t], z0, z1);
            sa = add2(sa, pk(ex2(z0 - ma), ex2(z1 - ma)));
          }
        }
        if (mb != -INFINITY) {
#pragma unroll
          for (int t = 0; t < kSmallGroup; ++t) {
            float z0, z1;
            upk(zb[t], z0, z1);
            sb = add2(sb, pk(ex2(z0 - mb), ex2(z1 - mb)));
          }
        }
      }
      float s0, s1;
      upk(sa, s0, s1);
      float suma = s0 + s1;
      upk(sb, s0, s1);
      float sumb = s0 + s1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float mao = __shfl_xor_sync(0xffffffffu, ma, o);
        const float sao = __shfl_xor_sync(0xffffffffu, suma, o);
        const float mbo = __shfl_xor_sync(0xffffffffu, mb, o);
        const float sbo = __shfl_xor_sync(0xffffffffu, sumb, o);
        merge_max_sum(ma, suma, mao, sao);
        merge_max_sum(mb, sumb, mbo, sbo);
      }
      // lane 0: row i, lane 1: row i2 (log2 of the sum in fp32: 2^-23 relative on a value
      // below ~25, ~3e-6 log2 units, far below the potentials' fp32 rounding; the rest in
      // double as the other passes do)
      const int row = lane == 0 ? i : i2;
      float hnew = 0.0f;
      if (lane < 2) {
        const double lse2 = lane == 0 ? static_cast<double>(ma) + static_cast<double>(log2f(suma))
                                      : static_cast<double>(mb) + static_cast<double>(log2f(sumb));
        const float pot = static_cast<float>(-lse2 * S.inv_kappa);
        if (lane == 0 || i2 != i) potr[row] = pot;
        hnew = small_bias(S.kappa, pot, R[D * rpad + row]);
      }
      // the new biases into every CTA of the cluster: lane c < csize stores to CTA c
      const float h0 = __shfl_sync(0xffffffffu, hnew, 0);
      const float h1 = __shfl_sync(0xffffffffu, hnew, 1);
      if (lane < static_cast<int>(csize)) {
        st_cluster(hr + i, static_cast<unsigned>(lane), h0);
        if (i2 != i) st_cluster(hr + i2, static_cast<unsigned>(lane), h1);
      }
    }
    // every row's potential and bias of this half-iteration written and visible to the
    // whole cluster, and every CTA done reading the key biases it used
    cluster_barrier();
  }
}

}  // namespace fs
