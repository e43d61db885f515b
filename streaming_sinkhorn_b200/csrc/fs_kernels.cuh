// fs_kernels.cuh -- CUDA kernels of the streaming log-domain Sinkhorn passes (sm_100a).
//
// One pass evaluates, for every query row i, the base-2 log-sum-exp over all key
// columns j of
//     z_ij = H_j - kappa |x_i - y_j|^2,   kappa = log2(e) / eps,   H_j = kappa g_j + log2 b_j,
// so that the f-update of the log-domain iteration (FlashSinkhorn summary, Methodology
// section 1) is F(g)_i = -LSE2_j(z_ij) / kappa. The same pass with the roles of the clouds
// swapped is the g-update. The squared distance is taken as a direct difference of the
// float32 input coordinates: its rounding error is relative to the local distances and
// potentials, where the expanded |x|^2 + |y|^2 - 2 x.y form loses precision in proportion to
// the squared distance from the origin (which over a few hundred slowly mixing iterations
// moves outlying potentials by more than 1e-4).
//
// Layout in HBM. Each cloud is stored once as "packed keys": point pairs (2p, 2p+1)
// share KP floats laid out as [c0 c0' c1 c1' ... c_{D-1} c_{D-1}' H H' pad], i.e. every
// coordinate (and the bias H) of the two points sits side by side so that one 64-bit
// register holds the same component of two columns, ready for the packed fp32x2 ops.
// The pair count is padded to a multiple of 128 with zero coordinates and H = kLogZero,
// which contribute nothing.
//
// A CTA owns NT*R query rows (R rows per thread, kept in registers) and streams one
// contiguous range of key pairs through shared memory with TMA bulk copies
// (kStages-deep ring, mbarrier completion). Each thread runs an online max/sum over its
// rows. The running offset m_i is folded into the distance accumulator,
//     t_ij = H_j - kappa (m_i / kappa + sum_k (x_ik - y_jk)^2) = z_ij - m_i,
// so a column pair costs d packed subtracts, d + 1 packed FMAs, two MUFU ex2 and one packed
// accumulate. Per group of G key pairs the row max of t is taken first and the running sum
// is rescaled only when it exceeds the offset by more than kLazyThr (terms then stay below
// 2^kLazyThr). When the key range is split over several CTAs, each writes its
// (max, sum[, weighted differences]) partial and a combine kernel merges them with a
// second-level LSE.
#pragma once

#include <cfloat>
#include <cmath>
#include "fs_device.cuh"
#include "fs_sort.cuh"

namespace fs {

// Floats per packed key pair for padded dimension D: 2(D+1) rounded up to 4.
__host__ __device__ constexpr int key_pair_floats(int D) { return ((2 * (D + 1) + 3) / 4) * 4; }

constexpr int kStages = 3;
constexpr float kLazyThr = 8.0f;
constexpr int kPairPad = 128;  // key pairs are padded to a multiple of this
// A group whose largest exponent is below this holds only zero-weight or padding
// columns; it never sets the running offset.
constexpr float kEmptyCut = -1.0e29f;

enum PassKind : int { kPot = 0, kMarg = 1, kGrad = 2 };

struct PassParams {
  const float* keys;        // streamed cloud, packed
  float* qkeys;             // query cloud, packed (coordinates read; H written by kPot)
  int64_t n_rows;           // real number of query rows
  int64_t key_pairs;        // padded key pair count
  int64_t pairs_per_split;  // key pairs per split (multiple of tile_pairs)
  int32_t tile_pairs;       // key pairs per shared-memory stage
  int32_t n_splits;         // gridDim.y
  int64_t rows_pad;         // row stride of the partial arrays
  int32_t kind;             // PassKind
  int32_t d_real;           // true dimension (<= D)
  float kappa_f;            // log2(e) / eps
  float inv_kappa_f;        // eps ln 2
  double kappa;             // log2(e) / eps
  double eps_ln2;           // eps ln 2 = 1 / kappa
  const float* lw;          // log2 weights of the query cloud (kLogZero for zeros)
  const float* w;           // linear weights of the query cloud, or NULL
  float w_uniform;          // weight used when w == NULL
  const float* pot_in;      // kMarg: given potential of the query cloud
  float* pot_out;           // kPot: new potential of the query cloud
  float* marg_out;          // kMarg: plan marginal per row, or NULL
  float* grad_out;          // kGrad: (n_rows, d_real)
  double* acc;              // kMarg: [sum |r - w|, max |r - w|, sum r]
  float* part_m;            // partial offsets [split][rows_pad]
  float* part_l;            // partial sums    [split][rows_pad]
  float* part_a;            // partial weighted differences [split][D][rows_pad]
  unsigned* err;            // error word
  // tensor-core passes: the next pass's key bias hy_i = H_i - kappa |x_i|^2 of the query
  // cloud (written instead of the packed-key slot) and its centred squared norms
  float* hy_out;
  const float* nrm;
  // spatially sorted clouds: sorted row -> original index of the query cloud (NULL: identity)
  const int* perm;
  // block screening (potential passes after the first two)
  int32_t screen;           // 1: skip key tiles whose every term is provably negligible
  const float* key_box;     // [tile][2D]: bounding box of each 256-point key tile
  const float* key_hmax;    // [tile]: largest key bias H of each key tile
  const int* key_dmin;      // ordered int: smallest change of the key biases since the last pass
  const float* lse_prev;    // LSE2 of every query row in its previous pass (sorted order)
  float log2_keys;          // log2(number of keys)
  float* lse_out;           // kPot: LSE2 of every query row (sorted order)
  int* dmin_out;            // kPot: ordered int, smallest change of the H this pass writes
  unsigned long long* evaluated;  // pairs evaluated after screening
};

constexpr int kScreenTile = 256;      // points per screening tile (= kPairPad pairs)
constexpr int kScreenMaxTiles = 4096; // tiles one CTA can screen (list in shared memory)
constexpr float kSkipMargin = 150.0f; // skipped terms are below 2^-150 of the row's largest

// Offset of coordinate slot k (k == D is the bias H) of point i in packed keys.
template <int D>
__device__ __forceinline__ int64_t key_slot(int64_t i, int k) {
  return (i >> 1) * key_pair_floats(D) + 2 * k + (i & 1);
}

// ---- per-row completion, shared by the direct epilogue and the combine kernel -----------

// kPot: the new potential and the bias this row carries as a key into the next pass:
//   pot_i = -LSE2_i / kappa,   H_i = kappa pot_i + log2 w_i = log2 w_i - LSE2_i.
// Returns the change of the row's key bias (new - previous), for the screening bound.
template <int D>
__device__ __forceinline__ float finish_pot(const PassParams& P, int64_t i, double lse2) {
  const int64_t oi = P.perm ? P.perm[i] : i;
  P.pot_out[oi] = static_cast<float>(-lse2 * P.eps_ln2);
  if (P.lse_out) P.lse_out[i] = static_cast<float>(lse2);
  const double h = static_cast<double>(P.lw[i]) - lse2;
  if (P.hy_out) {
    P.hy_out[i] = static_cast<float>(h - P.kappa * static_cast<double>(P.nrm[i]));
    return 0.0f;
  }
  const int64_t slot = key_slot<D>(i, D);
  const float hn = static_cast<float>(h);
  const float delta = hn - P.qkeys[slot];
  P.qkeys[slot] = hn;
  return delta;
}

// kMarg: plan marginal r_i = w_i 2^(kappa pot_i + LSE2_i) = w_i exp((pot_i - F_i)/eps).
__device__ __forceinline__ void finish_marg(const PassParams& P, int64_t i, double lse2,
                                            double& dev, double& mass) {
  const int64_t oi = P.perm ? P.perm[i] : i;
  const double w = P.w ? static_cast<double>(P.w[oi]) : static_cast<double>(P.w_uniform);
  double r = 0.0;
  if (w > 0.0) r = w * exp2(P.kappa * static_cast<double>(P.pot_in[oi]) + lse2);
  if (P.marg_out) P.marg_out[oi] = static_cast<float>(r);
  dev = fabs(r - w);
  mass = r;
}

// kGrad: grad_i = 2 w_i (x_i - T_i) = 2 w_i sum_j p_ij (x_i - y_j) / sum_j p_ij.
__device__ __forceinline__ void finish_grad(const PassParams& P, int64_t i, const float* dsum,
                                            float l) {
  const int64_t oi = P.perm ? P.perm[i] : i;
  const float w = P.w ? P.w[oi] : P.w_uniform;
  const float s = 2.0f * w / l;
  for (int k = 0; k < P.d_real; ++k) P.grad_out[oi * P.d_real + k] = s * dsum[k];
}

// Warp-wide minimum of the bias changes, one atomic per warp (NaN never wins fminf).
__device__ __forceinline__ void reduce_dmin(float v, int* out) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0 && out) atomicMin(out, float_ord(v));
}

// Block-wide sum/max of the marginal deviations, then one atomic per block.
__device__ __forceinline__ void block_reduce_marg(double dev_sum, double dev_max, double mass,
                                                  double* acc) {
  __shared__ double sh[3][32];
  dev_sum = warp_sum(dev_sum);
  dev_max = warp_max(dev_max);
  mass = warp_sum(mass);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) {
    sh[0][wid] = dev_sum;
    sh[1][wid] = dev_max;
    sh[2][wid] = mass;
  }
  __syncthreads();
  if (wid == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    double s = lane < nw ? sh[0][lane] : 0.0;
    double mx = lane < nw ? sh[1][lane] : 0.0;
    double ms = lane < nw ? sh[2][lane] : 0.0;
    s = warp_sum(s);
    mx = warp_max(mx);
    ms = warp_sum(ms);
    if (lane == 0) {
      atomicAdd(&acc[0], s);
      atomic_max_nonneg(&acc[1], mx);
      atomicAdd(&acc[2], ms);
    }
  }
}

// ---- the fused streaming pass -------------------------------------------------------------

// Loads the packed components of key pair p of a shared-memory tile.
template <int D>
__device__ __forceinline__ void load_pair(const float* tile, int p, u64 (&comp)[key_pair_floats(D) / 2]) {
  constexpr int NV = key_pair_floats(D) / 4;
  const ulonglong2* pv = reinterpret_cast<const ulonglong2*>(tile + p * key_pair_floats(D));
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const ulonglong2 q = pv[v];
    comp[2 * v] = q.x;
    comp[2 * v + 1] = q.y;
  }
}

template <int D, int R, int NT, int G, bool GRAD, int MINB>
__global__ void __launch_bounds__(NT, MINB) lse_pass_kernel(const PassParams P) {
  constexpr int KP = key_pair_floats(D);
  constexpr int NA = GRAD ? D : 1;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ uint64_t bars[kStages];

  float* stages = reinterpret_cast<float*>(smem_raw);
  const int tid = threadIdx.x;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * (NT * R);
  const int split = blockIdx.y;
  const int64_t p_begin = static_cast<int64_t>(split) * P.pairs_per_split;
  int64_t p_end = p_begin + P.pairs_per_split;
  if (p_end > P.key_pairs) p_end = P.key_pairs;
  const int n_tiles = static_cast<int>((p_end - p_begin) / P.tile_pairs);
  const uint32_t stage_floats = static_cast<uint32_t>(P.tile_pairs) * KP;
  const uint32_t stage_bytes = stage_floats * 4u;
  const float* key_src = P.keys + p_begin * KP;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }

  // Row state: coordinates duplicated into both lanes of a packed register; the running
  // offset m (log2 units), `base` (m, or 0 while no column has set it) and mk = base/kappa
  // folded into the distance accumulator; the running sums L (two lanes: even and odd
  // columns) and, for the gradient, the weighted differences A = sum p (x - y).
  u64 X[R][D];
  float m[R], base[R];
  u64 mk[R], L[R];
  u64 A[R][NA];
  const u64 nkappa = pk(-P.kappa_f, -P.kappa_f);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t i = row0 + r * NT + tid;
#pragma unroll
    for (int k = 0; k < D; ++k) {
      const float c = (i < P.n_rows) ? P.qkeys[key_slot<D>(i, k)] : 0.0f;
      X[r][k] = pk(c, c);
    }
    m[r] = -INFINITY;
    base[r] = 0.0f;
    mk[r] = pk(0.0f, 0.0f);
    L[r] = pk(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < NA; ++k) A[r][k] = pk(0.0f, 0.0f);
  }

  // Block screening (sorted clouds). Every pass first processes an anchor tile: the key
  // tile whose exponents have the largest upper bound (its largest bias minus kappa times
  // the squared distance between the CTA's row box and the tile's box). The running offset
  // it leaves is a value some term of the row reaches, hence a lower bound on the row's
  // largest exponent; a potential pass with history also has the bound "previous LSE2 plus
  // the smallest change of the key biases, minus log2(#keys)" (the largest term is at least
  // the sum over the count). Every other tile whose upper bound lies more than kSkipMargin
  // below the smallest of those bounds over the CTA's rows is skipped: each omitted term is
  // under 2^-kSkipMargin of its row's largest. The kept tiles form a list in shared memory.
  __shared__ unsigned short tlist[kScreenMaxTiles];
  __shared__ unsigned smask[kScreenMaxTiles / 32];
  __shared__ int s_box[2 * D];
  __shared__ int s_mlb, s_count;
  __shared__ unsigned long long s_best;
  const bool screening = P.screen && P.tile_pairs == kScreenTile / 2 && n_tiles > 1 &&
                         n_tiles <= kScreenMaxTiles;
  const bool history = screening && P.lse_prev && P.key_dmin;
  const int64_t T0 = p_begin / (kScreenTile / 2);
  int n_work = n_tiles;
  // Upper bound of the exponents of key tile tt for any row of this CTA.
  auto tile_ub = [&](int tt) -> float {
    const float* bx = P.key_box + (T0 + tt) * 2 * D;
    float d2 = 0.0f;
#pragma unroll
    for (int k = 0; k < D; ++k) {
      const float gap =
          fmaxf(fmaxf(bx[k] - ord_float(s_box[D + k]), ord_float(s_box[k]) - bx[D + k]), 0.0f);
      d2 = fmaf(gap, gap, d2);
    }
    return P.key_hmax[T0 + tt] - P.kappa_f * d2;
  };
  if (screening) {
    if (tid < D) {
      s_box[tid] = 0x7FFFFFFF;
      s_box[D + tid] = static_cast<int>(0x80000000u);
    }
    if (tid == 0) {
      s_mlb = 0x7FFFFFFF;
      s_best = 0ull;
    }
    __syncthreads();
    float lo[D], hi[D];
#pragma unroll
    for (int k = 0; k < D; ++k) {
      lo[k] = INFINITY;
      hi[k] = -INFINITY;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = row0 + r * NT + tid;
      if (i < P.n_rows) {
#pragma unroll
        for (int k = 0; k < D; ++k) {
          float c0, c1;
          upk(X[r][k], c0, c1);
          lo[k] = fminf(lo[k], c0);
          hi[k] = fmaxf(hi[k], c0);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int k = 0; k < D; ++k) {
        lo[k] = fminf(lo[k], __shfl_xor_sync(0xffffffffu, lo[k], o));
        hi[k] = fmaxf(hi[k], __shfl_xor_sync(0xffffffffu, hi[k], o));
      }
    }
    if ((tid & 31) == 0) {
#pragma unroll
      for (int k = 0; k < D; ++k) {
        atomicMin(&s_box[k], float_ord(lo[k]));
        atomicMax(&s_box[D + k], float_ord(hi[k]));
      }
    }
    __syncthreads();
    // anchor: largest upper bound, ties to the lower tile (key = ordered ub, then ~index)
    unsigned long long best = 0ull;
    for (int tt = tid; tt < n_tiles; tt += NT) {
      const unsigned ub = static_cast<unsigned>(float_ord(tile_ub(tt))) ^ 0x80000000u;
      const unsigned long long key =
          (static_cast<unsigned long long>(ub) << 32) | static_cast<unsigned>(0xFFFF - tt);
      best = best > key ? best : key;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = best > other ? best : other;
    }
    if ((tid & 31) == 0) atomicMax(&s_best, best);
    __syncthreads();
    if (tid == 0) tlist[0] = static_cast<unsigned short>(0xFFFF - (s_best & 0xFFFFull));
    __syncthreads();
    n_work = 1;  // the anchor; the kept tiles are appended once it is processed
  } else {
    __syncthreads();
    if (tid == 0 && P.evaluated)
      atomicAdd(P.evaluated, static_cast<unsigned long long>(n_tiles) * P.tile_pairs * 2 * (R * NT));
  }
  auto tile_src = [&](int e) -> const float* {
    const int tt = screening ? static_cast<int>(tlist[e]) : e;
    return key_src + static_cast<int64_t>(tt) * stage_floats;
  };

  // Online max/sum of this thread's rows over one key tile in shared memory.
  auto process_tile = [&](const float* tile) {
    for (int pg = 0; pg < P.tile_pairs; pg += G) {
      u64 tv[R][G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        u64 comp[KP / 2];
        load_pair<D>(tile, pg + g, comp);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          u64 acc = mk[r];
#pragma unroll
          for (int k = 0; k < D; ++k) {
            const u64 dk = sub2(X[r][k], comp[k]);
            acc = fma2(dk, dk, acc);
          }
          tv[r][g] = fma2(nkappa, acc, comp[D]);  // H - kappa (m/kappa + |x - y|^2)
        }
      }
      // Group max; lazy rescale of the running sums (always on a row's first real group).
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float a0, a1;
        upk(tv[r][0], a0, a1);
        float mx = fmaxf(a0, a1);
#pragma unroll
        for (int g = 1; g < G; ++g) {
          upk(tv[r][g], a0, a1);
          mx = max3(mx, a0, a1);
        }
        const float mx_abs = mx + base[r];
        if (mx_abs > m[r] + kLazyThr && mx > kEmptyCut) {
          const float sc = ex2(m[r] - mx_abs);
          const u64 sc2 = pk(sc, sc);
          L[r] = mul2(L[r], sc2);
          if (GRAD) {
#pragma unroll
            for (int k = 0; k < NA; ++k) A[r][k] = mul2(A[r][k], sc2);
          }
          const u64 sh = pk(-mx, -mx);
#pragma unroll
          for (int g = 0; g < G; ++g) tv[r][g] = add2(tv[r][g], sh);
          m[r] = mx_abs;
          base[r] = mx_abs;
          const float q = mx_abs * P.inv_kappa_f;
          mk[r] = pk(q, q);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        u64 comp[KP / 2];
        if (GRAD) load_pair<D>(tile, pg + g, comp);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float t0, t1;
          upk(tv[r][g], t0, t1);
          const u64 e = pk(ex2(t0), ex2(t1));
          L[r] = add2(L[r], e);
          if (GRAD) {
#pragma unroll
            for (int k = 0; k < NA; ++k) A[r][k] = fma2(e, sub2(X[r][k], comp[k]), A[r][k]);
          }
        }
      }
    }
  };

  // After the anchor: the lower bounds, the screen of the other tiles, the list, and the
  // first copies of the kept tiles.
  auto screen_rest = [&]() {
    const int anchor = tlist[0];
    const float dmin = history ? ord_float(*P.key_dmin) : 0.0f;
    float mlb = INFINITY;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = row0 + r * NT + tid;
      if (i < P.n_rows) {
        float b = m[r];
        if (history) b = fmaxf(b, P.lse_prev[i] + dmin - P.log2_keys);
        mlb = fminf(mlb, b);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mlb = fminf(mlb, __shfl_xor_sync(0xffffffffu, mlb, o));
    const int nwords = (n_tiles + 31) / 32;
    for (int w = tid; w < nwords; w += NT) smask[w] = 0u;
    if ((tid & 31) == 0) atomicMin(&s_mlb, float_ord(mlb));
    __syncthreads();
    const float mlb_min = ord_float(s_mlb);
    for (int tt = tid; tt < n_tiles; tt += NT) {
      if (tt != anchor && tile_ub(tt) >= mlb_min - kSkipMargin)
        atomicOr(&smask[tt >> 5], 1u << (tt & 31));
    }
    __syncthreads();
    if (tid < 32) {
      int running = 1;  // slot 0 holds the anchor
      for (int w0 = 0; w0 < nwords; w0 += 32) {
        const int w = w0 + tid;
        unsigned word = w < nwords ? smask[w] : 0u;
        const int cnt = __popc(word);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += v;
        }
        int pos = running + incl - cnt;
        while (word) {
          const int bit = __ffs(word) - 1;
          tlist[pos++] = static_cast<unsigned short>(w * 32 + bit);
          word &= word - 1u;
        }
        running += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (tid == 0) {
        s_count = running;
        if (P.evaluated)
          atomicAdd(P.evaluated, static_cast<unsigned long long>(running) * kScreenTile * (R * NT));
      }
    }
    __syncthreads();
    n_work = s_count;
    if (tid == 0) {
      for (int e = 1; e < kStages && e < n_work; ++e) {
        mbar_expect_tx(&bars[e], stage_bytes);
        bulk_g2s(stages + e * stage_floats, tile_src(e), stage_bytes, &bars[e]);
      }
    }
  };

  if (tid == 0) {
    for (int s = 0; s < kStages && s < n_work; ++s) {
      mbar_expect_tx(&bars[s], stage_bytes);
      bulk_g2s(stages + s * stage_floats, tile_src(s), stage_bytes, &bars[s]);
    }
  }

  // One CTA barrier per tile: after it every thread has finished the previous tile, so its
  // stage can be refilled, and a timed-out wait anywhere in the CTA is visible to all.
  int t = 0;
  bool aborted = false;
  for (; t < n_work; ++t) {
    const int st = t % kStages;
    const uint32_t parity = static_cast<uint32_t>(t / kStages) & 1u;
    const bool ok = mbar_wait_bounded(&bars[st], parity);
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    if (tid == 0 && t >= 1 && t - 1 + kStages < n_work) {
      const int ps = (t - 1) % kStages;
      fence_proxy_async_smem();
      mbar_expect_tx(&bars[ps], stage_bytes);
      bulk_g2s(stages + ps * stage_floats, tile_src(t - 1 + kStages), stage_bytes, &bars[ps]);
    }
    process_tile(stages + st * stage_floats);
    if (screening && t == 0) screen_rest();
  }

  if (aborted) {
    // Record the timeout, let this CTA's own copies still in flight land (bounded), leave.
    // Tiles t .. t + kStages - 2 were issued (tile t + kStages - 1 is issued only after the
    // barrier of tile t, which was not passed).
    if (tid == 0) {
      atomicOr(P.err, kErrTimeout);
      for (int u = t; u < n_work && u < t + kStages - 1; ++u)
        (void)mbar_wait_bounded(&bars[u % kStages], static_cast<uint32_t>(u / kStages) & 1u);
    }
    return;
  }

  if (P.n_splits == 1) {
    double dev_sum = 0.0, dev_max = 0.0, mass = 0.0;
    float dmin = INFINITY;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = row0 + r * NT + tid;
      if (i >= P.n_rows) continue;
      float l0, l1;
      upk(L[r], l0, l1);
      const float l = l0 + l1;
      if (GRAD) {
        float a[NA];
#pragma unroll
        for (int k = 0; k < NA; ++k) {
          float a0, a1;
          upk(A[r][k], a0, a1);
          a[k] = a0 + a1;
        }
        finish_grad(P, i, a, l);
      } else {
        const double lse2 = static_cast<double>(m[r]) + log2(static_cast<double>(l));
        if (P.kind == kPot) {
          dmin = fminf(dmin, finish_pot<D>(P, i, lse2));
        } else {
          double dv, ms;
          finish_marg(P, i, lse2, dv, ms);
          dev_sum += dv;
          dev_max = fmax(dev_max, dv);
          mass += ms;
        }
      }
    }
    if (!GRAD && P.kind == kMarg) block_reduce_marg(dev_sum, dev_max, mass, P.acc);
    if (!GRAD && P.kind == kPot) reduce_dmin(dmin, P.dmin_out);
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = row0 + r * NT + tid;
      if (i >= P.n_rows) continue;
      float l0, l1;
      upk(L[r], l0, l1);
      const int64_t o = static_cast<int64_t>(split) * P.rows_pad + i;
      P.part_m[o] = m[r];
      P.part_l[o] = l0 + l1;
      if (GRAD) {
#pragma unroll
        for (int k = 0; k < NA; ++k) {
          float a0, a1;
          upk(A[r][k], a0, a1);
          P.part_a[(static_cast<int64_t>(split) * D + k) * P.rows_pad + i] = a0 + a1;
        }
      }
    }
  }
}

// Second-level LSE over the split partials of each row, then the row completion. A split
// whose columns were all zero-weight or padding left m = -inf and sum 0 and drops out.
template <int D, bool GRAD>
__global__ void __launch_bounds__(256) combine_kernel(const PassParams P) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  double dev = 0.0, mass = 0.0;
  float dmin = INFINITY;
  if (i < P.n_rows) {
    float mx = -INFINITY;
    for (int s = 0; s < P.n_splits; ++s) mx = fmaxf(mx, P.part_m[s * P.rows_pad + i]);
    double l = 0.0;
    float a[GRAD ? D : 1];
    if (GRAD) {
      for (int k = 0; k < D; ++k) a[k] = 0.0f;
    }
    for (int s = 0; s < P.n_splits; ++s) {
      const int64_t o = s * P.rows_pad + i;
      const float pm = P.part_m[o];
      if (pm == -INFINITY) continue;
      const float w = ex2(pm - mx);
      l += static_cast<double>(P.part_l[o]) * w;
      if (GRAD) {
        for (int k = 0; k < D; ++k) a[k] += P.part_a[(static_cast<int64_t>(s) * D + k) * P.rows_pad + i] * w;
      }
    }
    if (GRAD) {
      finish_grad(P, i, a, static_cast<float>(l));
    } else {
      const double lse2 = static_cast<double>(mx) + log2(l);
      if (P.kind == kPot) {
        dmin = finish_pot<D>(P, i, lse2);
      } else {
        finish_marg(P, i, lse2, dev, mass);
      }
    }
  }
  if (!GRAD && P.kind == kMarg) block_reduce_marg(dev, dev, mass, P.acc);
  if (!GRAD && P.kind == kPot) reduce_dmin(dmin, P.dmin_out);
}

// ---- preparation kernels --------------------------------------------------------------

// Flags bit 1 for a non-finite coordinate.
__global__ void __launch_bounds__(256) check_coords_kernel(const float* pts, int64_t count,
                                                           unsigned* flags) {
  int bad = 0;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < count;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x)
    bad |= !isfinite(pts[j]);
  bad = warp_or(bad);
  if ((threadIdx.x & 31) == 0 && bad) atomicOr(flags, 1u);
}

// Weight sum (float64); flags bit 2 for a negative or non-finite weight.
__global__ void __launch_bounds__(256) reduce_weights_kernel(const float* w, int64_t count,
                                                             double* sum, unsigned* flags) {
  double s = 0.0;
  int bad = 0;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < count;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = w[j];
    bad |= !(v >= 0.0f) || isinf(v);
    s += v;
  }
  s = warp_sum(s);
  bad = warp_or(bad);
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(sum, s);
    if (bad) atomicOr(flags, 2u);
  }
}

// Flags bit 4 for a non-finite entry of a given potential.
__global__ void __launch_bounds__(256) check_finite_kernel(const float* v, int64_t count,
                                                           unsigned* flags) {
  int bad = 0;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < count;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x)
    bad |= !isfinite(v[j]);
  bad = warp_or(bad);
  if ((threadIdx.x & 31) == 0 && bad) atomicOr(flags, 4u);
}

// Packed keys (input coordinates, bias slot left to key_bias_kernel) and log2 weights for
// all padded points of one cloud.
template <int D>
__global__ void __launch_bounds__(256) pack_kernel(const float* pts, int64_t count, int32_t d_real,
                                                   const float* w, float w_uniform,
                                                   const int* perm, float* keys, float* lw,
                                                   int64_t pairs_pad) {
  constexpr int KP = key_pair_floats(D);
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= 2 * pairs_pad) return;
  const int64_t base = (j >> 1) * KP + (j & 1);
  if (j < count) {
    const int64_t src = perm ? perm[j] : j;  // slot j holds point perm[j]
#pragma unroll
    for (int k = 0; k < D; ++k) keys[base + 2 * k] = k < d_real ? pts[src * d_real + k] : 0.0f;
    const float wj = w ? w[src] : w_uniform;
    lw[j] = wj > 0.0f ? static_cast<float>(log2(static_cast<double>(wj))) : kLogZero;
  } else {
#pragma unroll
    for (int k = 0; k < D; ++k) keys[base + 2 * k] = 0.0f;
    keys[base + 2 * D] = kLogZero;
    lw[j] = kLogZero;
  }
  // zero the padding floats after the bias slot
#pragma unroll
  for (int k = 2 * D + 2; k < KP; k += 2) keys[base + k] = 0.0f;
}

// Key bias of every real point: H_j = kappa pot_j + log2 w_j (pot = 0 if NULL).
template <int D>
__global__ void __launch_bounds__(256) key_bias_kernel(float* keys, int64_t count, const float* pot,
                                                       const int* perm, const float* lw,
                                                       double kappa) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= count) return;
  const double p = pot ? static_cast<double>(pot[perm ? perm[j] : j]) : 0.0;
  keys[key_slot<D>(j, D)] = static_cast<float>(kappa * p + static_cast<double>(lw[j]));
}

// <v, w> in float64 (w NULL = uniform weight wu).
__global__ void __launch_bounds__(256) dot_kernel(const float* v, const float* w, float wu,
                                                  int64_t count, double* out) {
  double s = 0.0;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < count;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x)
    s += static_cast<double>(v[j]) * static_cast<double>(w ? w[j] : wu);
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) atomicAdd(out, s);
}

// cost = <f,a> + <g,b> - eps * (plan mass - m_a m_b)
__global__ void cost_finish_kernel(const double* fa, const double* gb, const double* mass,
                                   double eps, double mamb, double* out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) out[0] = fa[0] + gb[0] - eps * (mass[0] - mamb);
}

__global__ void residual_finish_kernel(const double* row_acc, const double* col_acc, double* out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    out[0] = row_acc[0];
    out[1] = row_acc[1];
    out[2] = col_acc[0];
    out[3] = col_acc[1];
  }
}

}  // namespace fs
