// fs_small.cuh -- small problems solved in one launch on a thread-block cluster (sm_100a).
//
// A fixed-count alternating solve (SinkSLOT README, API Reference: variant "alternating",
// stop_mode "fixed") of a problem with a few million pairs costs a few microseconds of
// exponentials per half-iteration, less than the launches, drains and merges of the
// streaming passes around it. Here one cluster of up to 16 CTAs runs every iteration in a
// single kernel: every CTA stages both clouds (coordinate-major) with their log2 weights in
// shared memory once; each half-iteration it refreshes the key biases
// H_j = kappa pot_j + log2 w_j from the potentials just written, its warps take rows in turn
// (the 32 lanes of a warp split a row's keys, two keys per packed fp32x2 operation and 16
// independent exponentials per step, and merge their (max, sum) pairs by shuffles), each
// row's new potential goes to global memory, and the CTAs meet at a
// hardware cluster barrier (release / acquire at cluster scope) before the next
// half-iteration reads them. The barrier cannot wait forever: every CTA of the cluster runs
// the same number of half-iterations and no CTA leaves early.
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
constexpr int kSmallGroup = 8;  // key pairs per lane per step (16 independent exponentials)
__host__ __device__ constexpr int64_t small_pad(int64_t count) {
  return (count + 64 * kSmallGroup - 1) / (64 * kSmallGroup) * (64 * kSmallGroup);
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
// weights, padded counts) and the biases of the current key cloud.
__host__ __device__ inline size_t small_smem_bytes(int64_t n, int64_t m, int D) {
  const int64_t np = small_pad(n), mp = small_pad(m);
  return static_cast<size_t>((np + mp) * (D + 1) + (np > mp ? np : mp)) * sizeof(float);
}

template <int D>
__global__ void __launch_bounds__(kSmallThreads) small_solve_kernel(const SmallParams S) {
  extern __shared__ __align__(16) float sm[];
  const int np = static_cast<int>(small_pad(S.n)), mp = static_cast<int>(small_pad(S.m));
  float* sx = sm;                       // x: [D][np] coordinates, then [np] log2 a
  float* sy = sx + (D + 1) * np;        // y: [D][mp], then [mp] log2 b
  float* hb = sy + (D + 1) * mp;        // biases H_j of the current key cloud
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
  }
  __syncthreads();
  const u64 nkap = pk(-static_cast<float>(S.kappa), -static_cast<float>(S.kappa));
  for (int h = 0; h < 2 * S.n_iters; ++h) {
    const bool rows_x = (h & 1) == 0;  // f-update first, then the g-update
    const float* R = rows_x ? sx : sy;
    const float* K = rows_x ? sy : sx;
    const int nr = rows_x ? S.n : S.m, nk = rows_x ? S.m : S.n;
    const int rpad = rows_x ? np : mp, kpad = rows_x ? mp : np;
    const float* potk = rows_x ? (h == 0 ? S.g_init : S.g) : S.f;  // NULL: zero potential
    float* potr = rows_x ? S.f : S.g;
    // 1. the key biases H_j = kappa pot_j + log2 w_j from the potentials of the previous
    //    half-iteration (read past L1: other CTAs of the cluster wrote them)
#pragma unroll 4
    for (int j = tid; j < kpad; j += kSmallThreads) {
      const float lw = K[D * kpad + j];
      float hj = kLogZero;
      if (j < nk && lw > kLogZero) {
        const double pj = potk ? static_cast<double>(__ldcg(potk + j)) : 0.0;
        hj = static_cast<float>(S.kappa * pj + static_cast<double>(lw));
      }
      hb[j] = hj;
    }
    __syncthreads();
    // 2. rows of this CTA, one warp per row; a lane takes key pairs lane + 32 t, kSmallGroup
    //    at a time, in packed fp32x2 arithmetic, and rescales its running sum only when a
    //    group's maximum exceeds its offset by more than kLazyThr
    const int stride = static_cast<int>(csize) * kSmallWarps;
    const u64* kc[D];
#pragma unroll
    for (int k = 0; k < D; ++k) kc[k] = reinterpret_cast<const u64*>(K + k * kpad);
    const u64* hv = reinterpret_cast<const u64*>(hb);
    for (int i = static_cast<int>(crank) * kSmallWarps + warp; i < nr; i += stride) {
      u64 xi[D];
#pragma unroll
      for (int k = 0; k < D; ++k) {
        const float c = R[k * rpad + i];
        xi[k] = pk(c, c);
      }
      float m = -INFINITY;
      u64 s2 = pk(0.0f, 0.0f);
      for (int q0 = lane; q0 < kpad / 2; q0 += 32 * kSmallGroup) {
        u64 z[kSmallGroup];
        float gmax = -INFINITY;
#pragma unroll
        for (int t = 0; t < kSmallGroup; ++t) {
          const int q = q0 + 32 * t;
          u64 acc = pk(0.0f, 0.0f);
#pragma unroll
          for (int k = 0; k < D; ++k) {
            const u64 dk = sub2(xi[k], kc[k][q]);
            acc = fma2(dk, dk, acc);
          }
          z[t] = fma2(nkap, acc, hv[q]);
          float z0, z1;
          upk(z[t], z0, z1);
          gmax = max3(gmax, z0, z1);
        }
        if (gmax > m + kLazyThr && gmax > kEmptyCut) {
          const float sc = m == -INFINITY ? 0.0f : ex2(m - gmax);
          s2 = mul2(s2, pk(sc, sc));
          m = gmax;
        }
        if (m != -INFINITY) {
#pragma unroll
          for (int t = 0; t < kSmallGroup; ++t) {
            float z0, z1;
            upk(z[t], z0, z1);
            s2 = add2(s2, pk(ex2(z0 - m), ex2(z1 - m)));
          }
        }
      }
      float s0, s1;
      upk(s2, s0, s1);
      float s = s0 + s1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
        const float so = __shfl_xor_sync(0xffffffffu, s, o);
        merge_max_sum(m, s, mo, so);
      }
      if (lane == 0) {
        // log2 of s in fp32 (2^-23 relative on a value below ~25: ~3e-6 log2 units, far
        // below the potentials' fp32 rounding), the rest in double as the other passes do
        const double lse2 = static_cast<double>(m) + static_cast<double>(log2f(s));
        potr[i] = static_cast<float>(-lse2 * S.inv_kappa);
      }
    }
    // 3. every potential of this half-iteration written and visible to the whole cluster,
    //    and every CTA done with its key biases
    cluster_barrier();
  }
}

}  // namespace fs
