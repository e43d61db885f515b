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
// The same with NP payload channels after the bias: [c0 c0' .. h h' p0 p0' .. pad].
__host__ __device__ constexpr int pair_floats(int D, int NP) {
  return ((2 * (D + 1 + NP) + 3) / 4) * 4;
}

// What a pass accumulates next to its row sums (the weights e = 2^(z - m)):
//   kModeLse  nothing (potential and marginal passes)
//   kModeGrad sum e (y' - x')                                     (gradient)
//   kModePay  sum e p_c over NP key payload channels               (transport products)
//   kModeDiff sum e (p_0 + (y' - x').v_i) (y' - x'), v_i per row   (Hessian-vector product)
enum PassMode : int { kModeLse = 0, kModeGrad = 1, kModePay = 2, kModeDiff = 3 };

constexpr int kStages = 3;
constexpr float kLazyThr = 8.0f;
constexpr int kPairPad = 128;  // key pairs are padded to a multiple of this
// A group whose largest exponent is below this holds only zero-weight or padding
// columns; it never sets the running offset.
constexpr float kEmptyCut = -1.0e29f;

// kLse: the row's LSE2 only (to lse_out), the fixed offset of a tensor-core apply pass.
enum PassKind : int { kPot = 0, kMarg = 1, kGrad = 2, kLse = 3 };

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
  // block screening (sorted clouds): the inputs of screen_kernel
  const float* key_box;     // [2D][key_tiles]: box of each 256-point key tile (lo, then hi)
  const float* key_hmax;    // [key_tiles]: largest key bias H of each key tile
  const float* key_sbox;    // [2D][key_supers]: the same for runs of kSuper tiles
  const float* key_shmax;   // [key_supers]
  int32_t key_tiles, key_supers;
  const int* key_dmin;      // ordered int: smallest change of the key biases since the last
                            // pass, or NULL (no history bound)
  const float* lse_prev;    // LSE2 of every query row in its previous pass (sorted order)
  float log2_keys;          // log2(number of keys)
  float skip_margin;        // log2 units below a row's lower bound under which tiles drop
  float* lse_out;           // kPot, kLse (and kMarg when set): LSE2 of every query row
                            // (sorted order)
  int* dmin_out;            // kPot: ordered int, smallest change of the H this pass writes
  unsigned long long* evaluated;  // pairs evaluated (after screening)
  // queue mode (screened passes): kept-tile bit masks and the unit plan
  const unsigned* kmask;    // [row block][mask_words], or NULL for split mode
  int32_t mask_words;       // 32-tile words per row block
  int32_t rb_rows;          // rows of a row block (R * NT of the pass)
  const int* kcount;        // [row block] kept tiles
  const int* unit_start;    // [row block + 1] first unit of each row block
  const int* unit_rb;       // [unit] row block of each unit (launch order)
  const int* unit_j;        // [unit] its index among its row block's units
  const int* qscal;         // [0] tiles per unit C, [1] number of units U
  // anchor record of the screen: per query row (sorted order) the key (sorted order) that
  // gave its largest anchor exponent; anchor_mode 1 evaluates the anchor tiles and records
  // it, 2 evaluates only the recorded key (0: anchor tiles, no record)
  int* anchor_key;
  int32_t anchor_mode;
  // group skip (screened passes, D <= 3): the key cloud's 16-point group records and each
  // query row's threshold (written by the screen, sorted order), or NULL
  const float* gsum;
  float* row_thr;
  // 1: the launch sized each stage of the copy ring for a key tile and its group records
  // (set by the host for the screened launches of D <= 3 kernels only)
  int32_t group_recs;
  const unsigned* key_codes; // Morton codes of the key cloud in sorted order (key_count)
  const unsigned* row_codes; // Morton codes of the query cloud in sorted order
  int64_t key_count;         // real keys
  // symmetric (Jacobi) schedule: blend weight (0: plain update) and, for the pass whose
  // biases the other pass of the same iteration must not see yet, where to leave them
  float alpha;
  float* defer_h;           // kPot: new bias of every query row (sorted order), or NULL
  // transport products and the Hessian-vector product (kModePay, kModeDiff)
  const float* tile_keys;   // the streamed cloud with payload channels, or NULL (keys)
  const float* row_v;       // kModeDiff: v_i per query row, (n_rows, d_real), caller order
  float* acc_out;           // results, caller order: row i at acc_out + i * acc_stride
  int32_t acc_k;            // channels written (<= the kernel's channel count)
  int32_t acc_stride;
};

constexpr int kScreenTile = 256;  // points per screening tile (= kPairPad pairs)
constexpr int kSortMemoWords = 12;  // words of the sort record a workspace keeps
// Relative size, in log2 units, below which the omitted part of a row's sum is kept: the
// skip margin is kSkipBits + log2(number of keys) (the tolerance of the screening). 24 bits
// is the fp32 unit roundoff: the omitted mass is at most one rounding of the row's sum.
constexpr float kSkipBits = 24.0f;

// Offset of coordinate slot k (k == D is the bias H) of point i in packed keys.
template <int D>
__device__ __forceinline__ int64_t key_slot(int64_t i, int k) {
  return (i >> 1) * key_pair_floats(D) + 2 * k + (i & 1);
}

// ---- per-row completion, shared by the direct epilogue and the combine kernel -----------

// kPot: the new potential and the bias this row carries as a key into the next pass:
//   pot_i = -LSE2_i / kappa,   H_i = kappa pot_i + log2 w_i = log2 w_i - LSE2_i.
// Returns the change of the row's key bias (new - previous), for the screening bound.
// Symmetric schedule: pot_i = (1 - alpha) pot_prev_i + alpha F_i (pot_prev read from
// pot_out before it is overwritten) and H_i = kappa pot_i + log2 w_i; the bias goes to
// defer_h when the other pass of the iteration still needs the previous one (the change
// is then recorded when it is applied).
template <int D>
__device__ __forceinline__ float finish_pot(const PassParams& P, int64_t i, double lse2) {
  const int64_t oi = P.perm ? P.perm[i] : i;
  double pot = -lse2 * P.eps_ln2;
  double h = static_cast<double>(P.lw[i]) - lse2;
  if (P.alpha > 0.0f) {
    const double a = static_cast<double>(P.alpha);
    pot = (1.0 - a) * static_cast<double>(P.pot_out[oi]) + a * pot;
    h = P.kappa * pot + static_cast<double>(P.lw[i]);
  }
  P.pot_out[oi] = static_cast<float>(pot);
  if (P.lse_out) P.lse_out[i] = static_cast<float>(lse2);
  if (P.hy_out) {
    const float hy = static_cast<float>(h - P.kappa * static_cast<double>(P.nrm[i]));
    if (P.defer_h)
      P.defer_h[i] = hy;
    else
      P.hy_out[i] = hy;
    return 0.0f;
  }
  const float hn = static_cast<float>(h);
  if (P.defer_h) {
    P.defer_h[i] = hn;
    return 0.0f;
  }
  const int64_t slot = key_slot<D>(i, D);
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
  if (P.lse_out) P.lse_out[i] = static_cast<float>(lse2);
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

// kModePay / kModeDiff: out_i = mass_i * (sum_j e_ij acc_ij) / (sum_j e_ij), mass_i the row's
// plan mass: its weight w_i on the plan of (F(g), g) (pot_in NULL), else the plan marginal
// w_i 2^(kappa pot_i + LSE2_i) of the given potentials (as finish_marg).
__device__ __forceinline__ void finish_acc(const PassParams& P, int64_t i, const float* a,
                                           double l, double lse2) {
  const int64_t oi = P.perm ? P.perm[i] : i;
  const double w = P.w ? static_cast<double>(P.w[oi]) : static_cast<double>(P.w_uniform);
  double mass = w;
  if (P.pot_in) mass = w > 0.0 ? w * exp2(P.kappa * static_cast<double>(P.pot_in[oi]) + lse2) : 0.0;
  const double s = l > 0.0 ? mass / l : 0.0;
  for (int c = 0; c < P.acc_k; ++c) P.acc_out[oi * P.acc_stride + c] = static_cast<float>(s * a[c]);
}

// Warp-wide minimum of the bias changes, one atomic per warp (NaN never wins fminf).
__device__ __forceinline__ void reduce_dmin(float v, int* out) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0 && out) atomicMin(out, float_ord(v));
}

// Block-wide sum/max of the marginal deviations, then one atomic per block (none when acc is
// NULL: a pass that only wants the per-row marginals). Every thread of the block calls it.
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
    if (lane == 0 && acc) {
      atomicAdd(&acc[0], s);
      atomic_max_nonneg(&acc[1], mx);
      atomicAdd(&acc[2], ms);
    }
  }
}

// Second-level LSE of row i over its ns partials (slots s0 .. s0 + ns - 1, row offset off
// within a slot of `stride` rows), then the row's completion. The partials are read
// kMergeChunk at a time, all loads of a chunk issued before any is used, so that a row
// costs one memory round trip per chunk rather than one per partial. A partial whose
// columns were all zero-weight or padding left m = -inf and sum 0 and drops out.
constexpr int kMergeChunk = 4;
template <int D, int MODE, int NA>
__device__ __forceinline__ void merge_row(const PassParams& P, int64_t i, int64_t s0, int64_t ns,
                                          int64_t stride, int64_t off, double& dev_sum,
                                          double& dev_max, double& mass, float& dmin) {
  constexpr bool GRAD = MODE == kModeGrad;
  constexpr bool ACC = MODE != kModeLse;
  float mx = -INFINITY;
  double l = 0.0;
  float a[NA];
#pragma unroll
  for (int k = 0; k < NA; ++k) a[k] = 0.0f;
  for (int64_t c0 = s0; c0 < s0 + ns; c0 += kMergeChunk) {
    float pm[kMergeChunk], pl[kMergeChunk];
#pragma unroll
    for (int u = 0; u < kMergeChunk; ++u) {
      const bool ok = c0 + u < s0 + ns;
      const int64_t o = (c0 + u) * stride + off;
      pm[u] = ok ? P.part_m[o] : -INFINITY;
      pl[u] = ok ? P.part_l[o] : 0.0f;
    }
    float cm = mx;
#pragma unroll
    for (int u = 0; u < kMergeChunk; ++u) cm = fmaxf(cm, pm[u]);
    if (cm == -INFINITY) continue;
    if (cm > mx) {  // rescale what was merged so far to the new maximum
      const float sc = ex2(mx - cm);
      l *= sc;
#pragma unroll
      for (int k = 0; k < NA; ++k) a[k] *= sc;
      mx = cm;
    }
#pragma unroll
    for (int u = 0; u < kMergeChunk; ++u) {
      const float w = pm[u] == -INFINITY ? 0.0f : ex2(pm[u] - mx);
      l += static_cast<double>(pl[u]) * w;
      if (ACC && c0 + u < s0 + ns) {
#pragma unroll
        for (int k = 0; k < NA; ++k) a[k] += P.part_a[((c0 + u) * NA + k) * stride + off] * w;
      }
    }
  }
  const double lse2 = static_cast<double>(mx) + log2(l);
  if (GRAD) {
    finish_grad(P, i, a, static_cast<float>(l));
  } else if (ACC) {
    finish_acc(P, i, a, l, lse2);
  } else if (P.kind == kPot) {
    dmin = fminf(dmin, finish_pot<D>(P, i, lse2));
  } else if (P.kind == kLse) {
    P.lse_out[i] = static_cast<float>(lse2);
  } else {
    double dv, ms;
    finish_marg(P, i, lse2, dv, ms);
    dev_sum += dv;
    dev_max = fmax(dev_max, dv);
    mass += ms;
  }
}

// ---- the fused streaming pass -------------------------------------------------------------

// Loads the packed components of key pair p of a shared-memory tile.
template <int KP>
__device__ __forceinline__ void load_pair(const float* tile, int p, u64 (&comp)[KP / 2]) {
  constexpr int NV = KP / 4;
  const ulonglong2* pv = reinterpret_cast<const ulonglong2*>(tile + p * KP);
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const ulonglong2 q = pv[v];
    comp[2 * v] = q.x;
    comp[2 * v + 1] = q.y;
  }
}

// GS: the instance of the screened launches of D <= 3, with the group skip; the unscreened
// launches use the one without it (fewer registers in the hot loop).
template <int D, int R, int NT, int G, int MODE, int NP, int MINB, int ST, bool GS>
__global__ void __launch_bounds__(NT, MINB) lse_pass_kernel(const PassParams P) {
  constexpr int kStages = ST;  // depth of the copy ring
  constexpr bool GRAD = MODE == kModeGrad;
  constexpr bool ACC = MODE != kModeLse;   // accumulates more than the row sums
  constexpr int KP = pair_floats(D, NP);   // key tile layout (payload channels after H)
  constexpr int NA = (MODE == kModeGrad || MODE == kModeDiff) ? D : (MODE == kModePay ? NP : 1);
  static_assert(MODE != kModeDiff || NP == 1, "the difference mode reads one payload channel");
  constexpr int RB = R * NT;  // rows of one row block
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ uint64_t bars[kStages];
  __shared__ uint64_t rbar;  // group skip: the record slot's copies
  __shared__ int s_walk[2];

  float* stages = reinterpret_cast<float*>(smem_raw);
  const int tid = threadIdx.x;
  // The copy ring holds kStages key tiles; with the group skip (one-warp CTAs, D <= 3,
  // screened launches) one slot behind it holds the 16-point group records of the tile
  // being processed. They are read only by the group tests at the start of the tile, after
  // which the next tile's records are copied in, so one slot suffices and keeps the CTA's
  // shared memory at the ring's size plus 512 B.
  constexpr bool GT = GS && NT == 32 && D <= 3;
  static_assert(!GT || G * 2 == kGroupKeys, "a key-pair group of the pass is a record's group");
  static_assert(!GT || R <= 2, "a lane tests its rows in the two halves of a packed register");
  static_assert(!GT || ST == 2, "the records of tile t + 1 follow the copy of tile t + 1");
  const uint32_t tile_floats = static_cast<uint32_t>(P.tile_pairs) * KP;
  const bool recs = GT && P.group_recs != 0;
  const uint32_t tile_bytes = tile_floats * 4u;
  float* rslot = stages + kStages * tile_floats;

  // The work of this CTA: rows row0 .. row0 + RB and a list of key tiles. Split mode: the
  // tiles of column split blockIdx.y, in order. Queue mode (screened, sorted clouds): unit
  // blockIdx.x of the screening plan, i.e. the kept tiles with ordinals [k0, k0 + n_work)
  // of row block b, read from the row block's bit mask.
  const bool queue = P.kmask != nullptr;
  int64_t row0, unit;
  int n_work, n_units = 1;
  const float* key_src;
  const unsigned* mrow = nullptr;
  if (queue) {
    if (static_cast<int>(blockIdx.x) >= P.qscal[1]) return;  // past the plan's unit count
    // unit blockIdx.x is the j-th unit of row block b; its partials go to slot first + j
    const int b = P.unit_rb[blockIdx.x];
    const int j = P.unit_j[blockIdx.x];
    const int first = P.unit_start[b];
    n_units = P.unit_start[b + 1] - first;
    unit = first + j;
    const int C = P.qscal[0];
    const int k0 = j * C;
    n_work = min(C, P.kcount[b] - k0);
    row0 = static_cast<int64_t>(b) * RB;
    key_src = P.tile_keys ? P.tile_keys : P.keys;
    mrow = P.kmask + static_cast<int64_t>(b) * P.mask_words;
    // Locate ordinal k0: the mask word holding it and how many set bits of that word precede it.
    if (tid < 32) {
      int before = 0;
      bool found = false;
      for (int w0 = 0; w0 < P.mask_words && !found; w0 += 32) {
        const int w = w0 + tid;
        const int cnt = w < P.mask_words ? __popc(mrow[w]) : 0;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += v;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, before + incl > k0);
        if (hit) {
          const int lane = __ffs(hit) - 1;
          if (tid == lane) {
            s_walk[0] = w;
            s_walk[1] = k0 - (before + incl - cnt);
          }
          found = true;
        }
        before += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (!found && tid == 0) {  // inconsistent plan: no tile is read, the rows get no result
        s_walk[0] = -1;
        s_walk[1] = 0;
        atomicOr(P.err, kErrTimeout);
      }
    }
  } else {
    unit = blockIdx.y;
    row0 = static_cast<int64_t>(blockIdx.x) * RB;
    const int64_t p_begin = static_cast<int64_t>(blockIdx.y) * P.pairs_per_split;
    int64_t p_end = p_begin + P.pairs_per_split;
    if (p_end > P.key_pairs) p_end = P.key_pairs;
    n_work = static_cast<int>((p_end - p_begin) / P.tile_pairs);
    n_units = P.n_splits;
    key_src = (P.tile_keys ? P.tile_keys : P.keys) + p_begin * KP;
    if (tid == 0 && P.evaluated)
      atomicAdd(P.evaluated, static_cast<unsigned long long>(n_work) * P.tile_pairs * 2 * RB);
  }

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    if (recs) mbar_init(&rbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (queue && s_walk[0] < 0) n_work = 0;

  // Thread 0 issues the copies in order; in queue mode it walks the set bits of the mask
  // from the located start (the plan guarantees n_work of them; the walk stays inside the
  // row's words regardless and falls back to tile 0 if they run out).
  int walk_w = 0;
  unsigned walk_bits = 0u;
  if (queue && tid == 0 && n_work > 0) {
    walk_w = s_walk[0];
    walk_bits = mrow[walk_w];
    for (int s = 0; s < s_walk[1]; ++s) walk_bits &= walk_bits - 1u;
  }
  // Group skip: queue mode with the screen's row thresholds and the key cloud's records.
  const bool gtest = recs && queue && P.row_thr && P.gsum;
  int rtt0 = 0, rtt1 = 0;  // thread 0: the key tiles of the work items in flight, by parity
  // Issues the copy of work item e's key tile (thread 0).
  auto issue_tile = [&](int s, int e) {
    int tt = e;
    if (queue) {
      while (walk_bits == 0u && walk_w + 1 < P.mask_words) walk_bits = mrow[++walk_w];
      tt = walk_bits ? walk_w * 32 + __ffs(walk_bits) - 1 : 0;
      walk_bits &= walk_bits - 1u;
    }
    if (e & 1)
      rtt1 = tt;
    else
      rtt0 = tt;
    float* dst = stages + s * tile_floats;
    mbar_expect_tx(&bars[s], tile_bytes);
    bulk_g2s(dst, key_src + static_cast<int64_t>(tt) * tile_floats, tile_bytes, &bars[s]);
  };
  // Issues the copy of work item e's group records into the slot (thread 0; its key tile
  // has been issued).
  auto issue_recs = [&](int e) {
    const int tt = (e & 1) ? rtt1 : rtt0;
    mbar_expect_tx(&rbar, kTileGroupFloats * 4u);
    bulk_g2s(rslot, P.gsum + static_cast<int64_t>(tt) * kTileGroupFloats, kTileGroupFloats * 4u,
             &rbar);
  };

  // Row state: coordinates duplicated into both lanes of a packed register; the running
  // offset m (log2 units), `base` (m, or 0 while no column has set it) and mk = base/kappa
  // folded into the distance accumulator; the running sums L (two lanes: even and odd
  // columns) and, for the gradient, the weighted differences A = sum p (x - y).
  //
  // One-warp CTAs (CEN) use the centred expanded form instead. With c the centre of the
  // warp's row box, x' = x - c and y' = y - c,
  //   z - base = (H - kappa |y'|^2) - (base + kappa |x'|^2) + sum_k (2 kappa x'_k) y'_k,
  // so each tile is rewritten once in place to (y', H' = H - kappa |y'|^2), X holds
  // 2 kappa x', mk holds -(base + kappa |x'|^2), and a pair costs D + 1 packed operations
  // instead of 2D + 1. Centring keeps every magnitude at the scale of the row box and the
  // kept tiles around it, where the direct form's rounding also lives. The gradient
  // accumulates sum p (y' - x') term by term (x' recovered from X), not x' L - sum p y',
  // whose cancellation would cost digits when x is close to its barycentre.
  constexpr bool CEN = NT == 32;
  u64 X[R][D];
  float m[R], base[R];
  u64 mk[R], L[R];
  u64 A[R][NA];
  u64 V[R][MODE == kModeDiff ? D : 1];  // kModeDiff: the row's vector v_i, in both lanes
  float q[R];        // CEN: kappa |x'|^2
  u64 cpk[D];        // CEN: the centre, in both lanes
  u64 xb[GT ? D : 1];  // group skip: x of the thread's two rows (one per lane)
  u64 thr2 = pk(INFINITY, INFINITY);  // group skip: their thresholds
  // group skip: the warp's row box (lo, hi per coordinate) and its smallest threshold, in
  // shared memory (they are read once per tile)
  __shared__ float s_wbox[2 * 3 + 1];
  int groups_done = 0;  // group skip: 16-point groups this warp evaluated
  const u64 nkappa = pk(-P.kappa_f, -P.kappa_f);
  const u64 nhalf_ik = pk(-0.5f * P.inv_kappa_f, -0.5f * P.inv_kappa_f);  // X -> -x'
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
    if constexpr (MODE == kModeDiff) {
      const int64_t oi = i < P.n_rows ? (P.perm ? P.perm[i] : i) : -1;
#pragma unroll
      for (int k = 0; k < D; ++k) {
        const float v = (oi >= 0 && k < P.d_real) ? P.row_v[oi * P.d_real + k] : 0.0f;
        V[r][k] = pk(v, v);
      }
    }
  }
  if constexpr (CEN) {
#pragma unroll
    for (int k = 0; k < D; ++k) {
      float lo = INFINITY, hi = -INFINITY;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (row0 + r * NT + tid < P.n_rows) {
          float c0, c1;
          upk(X[r][k], c0, c1);
          lo = fminf(lo, c0);
          hi = fmaxf(hi, c0);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      }
      const float c = lo <= hi ? 0.5f * (lo + hi) : 0.0f;
      cpk[k] = pk(c, c);
      if constexpr (GT) {
        if (tid == 0) {
          s_wbox[k] = lo;
          s_wbox[3 + k] = hi;
        }
      }
    }
    if constexpr (GT) {
#pragma unroll
      for (int k = 0; k < D; ++k) {
        float c0, c1, d0, d1;
        upk(X[0][k], c0, c1);
        upk(X[R > 1 ? 1 : 0][k], d0, d1);
        xb[k] = pk(c0, d0);
      }
    }
    const float k2 = 2.0f * P.kappa_f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float s2 = 0.0f;
#pragma unroll
      for (int k = 0; k < D; ++k) {
        float c0, c1, cc, cd;
        upk(X[r][k], c0, c1);
        upk(cpk[k], cc, cd);
        const float xs = c0 - cc;
        s2 = fmaf(xs, xs, s2);
        X[r][k] = pk(k2 * xs, k2 * xs);
      }
      q[r] = P.kappa_f * s2;
      mk[r] = pk(-q[r], -q[r]);
    }
    if constexpr (GT) {
      if (gtest) {
        float t0 = INFINITY, t1 = INFINITY;  // rows past the end need nothing
        const int64_t i0 = row0 + tid, i1 = row0 + (R > 1 ? NT : 0) + tid;
        if (i0 < P.n_rows) t0 = P.row_thr[i0];
        if (R > 1 && i1 < P.n_rows) t1 = P.row_thr[i1];
        thr2 = pk(t0, t1);
        float wthr = fminf(t0, t1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wthr = fminf(wthr, __shfl_xor_sync(0xffffffffu, wthr, o));
        if (tid == 0) s_wbox[6] = wthr;
        __syncwarp();
      }
    }
  }
  // CEN: rewrite a tile in place to (y', H'); pairs are spread over the warp's lanes.
  // With the group skip, a run of 32 pairs (four groups) none of which is kept is left as it is.
  auto centre_tile = [&](float* tile, unsigned gm) {
    if constexpr (CEN) {
      for (int p = tid; p < P.tile_pairs; p += 32) {
        if (((gm >> ((p - tid) / G)) & 0xFu) == 0u) continue;
        u64 comp[KP / 2];
        load_pair<KP>(tile, p, comp);
        u64 s2 = pk(0.0f, 0.0f);
#pragma unroll
        for (int k = 0; k < D; ++k) {
          comp[k] = sub2(comp[k], cpk[k]);
          s2 = fma2(comp[k], comp[k], s2);
        }
        comp[D] = fma2(nkappa, s2, comp[D]);
        ulonglong2* pv = reinterpret_cast<ulonglong2*>(tile + p * KP);
#pragma unroll
        for (int v = 0; v < KP / 4; ++v) pv[v] = make_ulonglong2(comp[2 * v], comp[2 * v + 1]);
      }
      __syncwarp();
    }
  };

  // Group skip: bit g of the result is set when some row of the warp may need group g of the
  // tile (records in the slot, coordinates uncentred, as the screen tests them). Lane g < 16
  // first tests group g against the warp's row box and smallest threshold: a group that
  // fails fails every row's own test, which then runs, two groups at a time, on the others.
  auto group_mask = [&]() -> unsigned {
    unsigned gm = 0u;
    if constexpr (GT) {
      bool cand = false;
      if (tid < kTileGroupFloats / kGroupRecFloats) {
        const float4* r4 = reinterpret_cast<const float4*>(rslot + tid * kGroupRecFloats);
        const float4 ra = r4[0], rb = r4[1];  // lo0 lo1 lo2 hi0 | hi1 hi2 Hmax -
        const float glo[3] = {ra.x, ra.y, ra.z}, ghi[3] = {ra.w, rb.x, rb.y};
        float d2 = 0.0f;
#pragma unroll
        for (int k = 0; k < D; ++k) {
          const float gap = max3(glo[k] - s_wbox[3 + k], s_wbox[k] - ghi[k], 0.0f);
          d2 = fmaf(gap, gap, d2);
        }
        cand = rb.z - P.kappa_f * d2 >= s_wbox[6];
      }
      unsigned cm = __ballot_sync(0xffffffffu, cand);
      float h0, h1;
      upk(thr2, h0, h1);
      auto row_test = [&](int gi) -> bool {
        const float4* r4 = reinterpret_cast<const float4*>(rslot + gi * kGroupRecFloats);
        const float4 ra = r4[0], rb = r4[1];
        const float lo[3] = {ra.x, ra.y, ra.z}, hi[3] = {ra.w, rb.x, rb.y};
        u64 d2 = pk(0.0f, 0.0f);
#pragma unroll
        for (int k = 0; k < D; ++k) {
          float a0, a1, b0, b1;
          upk(sub2(pk(lo[k], lo[k]), xb[k]), a0, a1);
          upk(sub2(xb[k], pk(hi[k], hi[k])), b0, b1);
          const u64 gap = pk(max3(a0, b0, 0.0f), max3(a1, b1, 0.0f));
          d2 = fma2(gap, gap, d2);
        }
        float e0, e1;
        upk(d2, e0, e1);
        return rb.z - P.kappa_f * e0 >= h0 || rb.z - P.kappa_f * e1 >= h1;
      };
      while (cm) {
        const int g0 = __ffs(cm) - 1;
        cm &= cm - 1u;
        const int g1 = cm ? __ffs(cm) - 1 : g0;
        cm &= cm - 1u;
        const bool n0 = row_test(g0), n1 = row_test(g1);
        if (__any_sync(0xffffffffu, n0)) gm |= 1u << g0;
        if (__any_sync(0xffffffffu, n1)) gm |= 1u << g1;
      }
    }
    return gm;
  };

  // Online max/sum of this thread's rows over one key tile in shared memory. With the group
  // skip, a group of G key pairs is left out when for every row of the warp its upper bound
  // Hmax_g - kappa dist(x_i, box_g)^2 is below the row's threshold (the screen's lower bound
  // on the row's largest exponent minus the margin): each of its terms is then below
  // 2^-margin of the row's largest, as for the tiles the screen drops, and all keys left out
  // either way number at most M, so the omitted part of the row's sum stays below 2^-24 of it.
  auto process_tile = [&](const float* tile, unsigned gm) {
    for (int pg = 0; pg < P.tile_pairs; pg += G) {
      if ((gm >> (pg / G) & 1u) == 0u) continue;
      u64 tv[R][G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        u64 comp[KP / 2];
        load_pair<KP>(tile, pg + g, comp);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if constexpr (CEN) {
            u64 acc = add2(comp[D], mk[r]);  // H' - base - kappa |x'|^2
#pragma unroll
            for (int k = 0; k < D; ++k) acc = fma2(X[r][k], comp[k], acc);
            tv[r][g] = acc;
          } else {
            u64 acc = mk[r];
#pragma unroll
            for (int k = 0; k < D; ++k) {
              const u64 dk = sub2(X[r][k], comp[k]);
              acc = fma2(dk, dk, acc);
            }
            tv[r][g] = fma2(nkappa, acc, comp[D]);  // H - kappa (m/kappa + |x - y|^2)
          }
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
          if (ACC) {
#pragma unroll
            for (int k = 0; k < NA; ++k) A[r][k] = mul2(A[r][k], sc2);
          }
          const u64 sh = pk(-mx, -mx);
#pragma unroll
          for (int g = 0; g < G; ++g) tv[r][g] = add2(tv[r][g], sh);
          m[r] = mx_abs;
          base[r] = mx_abs;
          if constexpr (CEN) {
            const float nb = -(mx_abs + q[r]);
            mk[r] = pk(nb, nb);
          } else {
            const float qb = mx_abs * P.inv_kappa_f;
            mk[r] = pk(qb, qb);
          }
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        u64 comp[KP / 2];
        if (ACC) load_pair<KP>(tile, pg + g, comp);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float t0, t1;
          upk(tv[r][g], t0, t1);
          const u64 e = pk(ex2(t0), ex2(t1));
          L[r] = add2(L[r], e);
          if constexpr (MODE == kModeGrad) {
#pragma unroll
            for (int k = 0; k < NA; ++k)
              A[r][k] = CEN ? fma2(e, fma2(X[r][k], nhalf_ik, comp[k]), A[r][k])  // e (y' - x')
                            : fma2(e, sub2(X[r][k], comp[k]), A[r][k]);
          } else if constexpr (MODE == kModePay) {
#pragma unroll
            for (int c = 0; c < NA; ++c) A[r][c] = fma2(e, comp[D + 1 + c], A[r][c]);
          } else if constexpr (MODE == kModeDiff) {
            u64 dk[D];
            u64 w = comp[D + 1];  // p_0 + (y' - x').v_i
#pragma unroll
            for (int k = 0; k < D; ++k) {
              dk[k] = fma2(X[r][k], nhalf_ik, comp[k]);
              w = fma2(dk[k], V[r][k], w);
            }
            const u64 ew = mul2(e, w);
#pragma unroll
            for (int k = 0; k < D; ++k) A[r][k] = fma2(ew, dk[k], A[r][k]);
          }
        }
      }
    }  };

  if (tid == 0) {
    for (int s = 0; s < kStages && s < n_work; ++s) issue_tile(s, s);
    if (gtest && n_work > 0) issue_recs(0);
  }

  // One CTA barrier per tile: after it every thread has finished the previous tile, so its
  // stage can be refilled, and a timed-out wait anywhere in the CTA is visible to all.
  int t = 0;
  bool aborted = false;
  for (; t < n_work; ++t) {
    const int st = t % kStages;
    const uint32_t parity = static_cast<uint32_t>(t / kStages) & 1u;
    bool ok = mbar_wait_bounded(&bars[st], parity);
    if (gtest) ok = mbar_wait_bounded(&rbar, static_cast<uint32_t>(t) & 1u) && ok;
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    if (tid == 0 && t >= 1 && t - 1 + kStages < n_work) {
      const int ps = (t - 1) % kStages;
      fence_proxy_async_smem();
      issue_tile(ps, t - 1 + kStages);
    }
    unsigned gm = 0xffffffffu;
    if constexpr (GT) {
      if (gtest) {
        gm = group_mask();
        groups_done += __popc(gm);
        // every lane's reads of the slot are done (the votes above): the next records may
        // overwrite it; order those generic reads before the asynchronous copy
        __syncwarp();
        if (tid == 0 && t + 1 < n_work) {
          fence_proxy_async_smem();
          issue_recs(t + 1);
        }
      }
    }
    if constexpr (CEN) centre_tile(stages + st * tile_floats, gm);
    process_tile(stages + st * tile_floats, gm);
    // the stage was written by this (generic) proxy: order that before its next copy
    if constexpr (CEN) fence_proxy_async_smem();
  }
  if (queue && P.evaluated && tid == 0 && n_work > 0)
    atomicAdd(P.evaluated, gtest ? static_cast<unsigned long long>(groups_done) * kGroupKeys * RB
                                 : static_cast<unsigned long long>(n_work) * kScreenTile * RB);

  if (aborted) {
    // Record the timeout, let this CTA's own copies still in flight land (bounded), leave.
    // Tiles t .. t + kStages - 2 were issued (tile t + kStages - 1 is issued only after the
    // barrier of tile t, which was not passed).
    if (tid == 0) {
      atomicOr(P.err, kErrTimeout);
      for (int u = t; u < n_work && u < t + kStages - 1; ++u)
        (void)mbar_wait_bounded(&bars[u % kStages], static_cast<uint32_t>(u / kStages) & 1u);
      if (gtest) (void)mbar_wait_bounded(&rbar, static_cast<uint32_t>(t) & 1u);  // tile t's records
    }
    return;
  }

  // sum_j p_ij (x_i - y_j) of row r, component k (CEN accumulates its negative)
  auto diff_sum = [&](int r, int k) -> float {
    float a0, a1;
    upk(A[r][k], a0, a1);
    return CEN ? -(a0 + a1) : a0 + a1;
  };

  if (n_units == 1) {
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
        for (int k = 0; k < NA; ++k) a[k] = diff_sum(r, k);
        finish_grad(P, i, a, l);
      } else if (ACC) {
        float a[NA];
#pragma unroll
        for (int k = 0; k < NA; ++k) {
          float a0, a1;
          upk(A[r][k], a0, a1);
          a[k] = a0 + a1;
        }
        finish_acc(P, i, a, static_cast<double>(l),
                   static_cast<double>(m[r]) + log2(static_cast<double>(l)));
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
    if (!ACC && P.kind == kMarg) block_reduce_marg(dev_sum, dev_max, mass, P.acc);
    if (!ACC && P.kind == kPot) reduce_dmin(dmin, P.dmin_out);
  } else {
    // Partials of this unit: split mode at [split][rows_pad] (global row index), queue mode
    // at [unit][RB] (row index within the block).
    const int64_t pstride = queue ? RB : P.rows_pad;
    const int64_t poff = queue ? -row0 : 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = row0 + r * NT + tid;
      if (i >= P.n_rows) continue;
      float l0, l1;
      upk(L[r], l0, l1);
      const int64_t o = unit * pstride + poff + i;
      P.part_m[o] = m[r];
      P.part_l[o] = l0 + l1;
      if (ACC) {
#pragma unroll
        for (int k = 0; k < NA; ++k) {
          float a0, a1;
          upk(A[r][k], a0, a1);
          P.part_a[(unit * NA + k) * pstride + poff + i] = GRAD ? diff_sum(r, k) : a0 + a1;
        }
      }
    }
  }
}

// Second-level LSE over the partials of each row, then the row completion. Split mode: the
// n_splits partials at [split][rows_pad]. Queue mode: the units of the row's block at
// [unit][rb_rows]; a block with one unit was completed by the pass itself. The loads the
// row's completion will need are sent to L2 first, so they overlap the partials' loads.
template <int D, int MODE, int NA>
__global__ void __launch_bounds__(256) combine_kernel(const PassParams P) {
  constexpr bool ACC = MODE != kModeLse;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  double dev_sum = 0.0, dev_max = 0.0, mass = 0.0;
  float dmin = INFINITY;
  if (i < P.n_rows) {
    if (P.perm) prefetch_l2(P.perm + i);
    if (!ACC && P.kind == kPot) {
      prefetch_l2(P.lw + i);
      if (!P.hy_out && !P.defer_h) prefetch_l2(P.qkeys + key_slot<D>(i, D));
    }
    int64_t s0 = 0, ns = P.n_splits, stride = P.rows_pad, off = i;
    if (P.kmask) {
      const int64_t b = i / P.rb_rows;
      s0 = P.unit_start[b];
      ns = P.unit_start[b + 1] - s0;
      stride = P.rb_rows;
      off = i - b * P.rb_rows;
    }
    if (ns > 1 || !P.kmask)
      merge_row<D, MODE, NA>(P, i, s0, ns, stride, off, dev_sum, dev_max, mass, dmin);
  }
  if (!ACC && P.kind == kMarg) block_reduce_marg(dev_sum, dev_max, mass, P.acc);
  if (!ACC && P.kind == kPot) reduce_dmin(dmin, P.dmin_out);
}

// ---- preparation kernels --------------------------------------------------------------

// The splitmix64 output mixer (Steele, Lea and Flood, "Fast splittable pseudorandom number
// generators", 2014, with the "variant 13" constants of D. Stafford that Vigna's splitmix64
// uses): a bijective 64-bit mixer.
__device__ __forceinline__ unsigned long long mix64(unsigned long long z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  return z ^ (z >> 31);
}

// Flags bit 1 for a non-finite coordinate; adds a fingerprint of the coordinates (the sum
// over entries of mix64(index, bits), so it does not depend on the reduction order) to *hash.
__global__ void __launch_bounds__(256) check_coords_kernel(const float* pts, int64_t count,
                                                           unsigned* flags,
                                                           unsigned long long* hash) {
  int bad = 0;
  unsigned long long h = 0ull;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < count;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = pts[j];
    bad |= !isfinite(v);
    h += mix64((static_cast<unsigned long long>(j) << 32) ^ __float_as_uint(v));
  }
  bad = warp_or(bad);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) h += __shfl_xor_sync(0xffffffffu, h, o);
  if ((threadIdx.x & 31) == 0) {
    if (bad) atomicOr(flags, 1u);
    atomicAdd(hash, h);
  }
}

// The record of the last sort kept in a workspace (see prepare()).
struct SortMemo {
  unsigned long long v[kSortMemoWords];
};
__global__ void sort_memo_kernel(unsigned long long* memo, const SortMemo m) {
  if (threadIdx.x < kSortMemoWords) memo[threadIdx.x] = m.v[threadIdx.x];
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

// Key tiles with payload: coordinates and bias of every packed pair copied from the
// standard layout, then NP payload channels, pay[caller index * stride + c] for c < k (0
// beyond k and for padding points). One thread per point.
template <int D, int NP>
__global__ void __launch_bounds__(256) payload_keys_kernel(const float* keys, int64_t count,
                                                           int64_t pairs, const float* pay,
                                                           int k, int stride, const int* perm,
                                                           float* out) {
  constexpr int K0 = key_pair_floats(D), K1 = pair_floats(D, NP);
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= 2 * pairs) return;
  const int64_t p = j >> 1;
  const int e = static_cast<int>(j & 1);
  const float* src = keys + p * K0;
  float* dst = out + p * K1;
#pragma unroll
  for (int c = 0; c <= D; ++c) dst[2 * c + e] = src[2 * c + e];
  const int64_t oi = j < count ? (perm ? perm[j] : j) : -1;
#pragma unroll
  for (int c = 0; c < NP; ++c)
    dst[2 * (D + 1 + c) + e] = (oi >= 0 && c < k) ? pay[oi * stride + c] : 0.0f;
  for (int q = 2 * (D + 1 + NP) + e; q < K1; q += 2) dst[q] = 0.0f;
}

// Coarse stage: one cell per `cell_points` consecutive points of a sorted cloud (consecutive
// in Morton order, so spatially compact; cell_points <= 256): its mass sum_j w_j and its
// weighted centroid. One CTA per cell. A cell without mass takes the plain mean of its
// points (it then carries no weight).
template <int D>
__global__ void __launch_bounds__(256) cell_kernel(const float* keys, int64_t count, int32_t d_real,
                                                   const float* w, float w_uniform,
                                                   const int* perm, int cell_points,
                                                   float* cell_pts, float* cell_mass) {
  __shared__ double red[8][D + 2];
  __shared__ double pred[8][D];
  const int64_t c = blockIdx.x;
  const int64_t j = c * cell_points + threadIdx.x;
  const bool mine = static_cast<int>(threadIdx.x) < cell_points && j < count;
  double acc[D + 2];
#pragma unroll
  for (int k = 0; k < D + 2; ++k) acc[k] = 0.0;
  if (mine) {
    const int64_t oi = perm ? perm[j] : j;
    const double wj = w ? static_cast<double>(w[oi]) : static_cast<double>(w_uniform);
#pragma unroll
    for (int k = 0; k < D; ++k) acc[k] = wj * static_cast<double>(keys[key_slot<D>(j, k)]);
    acc[D] = wj;
    acc[D + 1] = 1.0;
  }
  double plain[D];
#pragma unroll
  for (int k = 0; k < D; ++k) plain[k] = mine ? static_cast<double>(keys[key_slot<D>(j, k)]) : 0.0;
#pragma unroll
  for (int k = 0; k < D + 2; ++k) acc[k] = warp_sum(acc[k]);
#pragma unroll
  for (int k = 0; k < D; ++k) plain[k] = warp_sum(plain[k]);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < D + 2; ++k) red[wid][k] = acc[k];
#pragma unroll
    for (int k = 0; k < D; ++k) pred[wid][k] = plain[k];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t[D + 2], q[D];
    for (int k = 0; k < D + 2; ++k) t[k] = 0.0;
    for (int k = 0; k < D; ++k) q[k] = 0.0;
    for (int r = 0; r < 8; ++r) {
      for (int k = 0; k < D + 2; ++k) t[k] += red[r][k];
      for (int k = 0; k < D; ++k) q[k] += pred[r][k];
    }
    const double mass = t[D], pts = t[D + 1];
    for (int k = 0; k < d_real; ++k)
      cell_pts[c * d_real + k] =
          static_cast<float>(mass > 0.0 ? t[k] / mass : (pts > 0.0 ? q[k] / pts : 0.0));
    cell_mass[c] = static_cast<float>(mass);
  }
}

// Debiased divergence: S = c[0] - c[1]/2 - c[2]/2.
__global__ void divergence_finish_kernel(const double* c, double* out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *out = c[0] - 0.5 * c[1] - 0.5 * c[2];
}

// grad -= (u + v) / 2 (the self problem's two one-sided gradients).
__global__ void __launch_bounds__(256) sub_half_sum_kernel(float* grad, const float* u,
                                                           const float* v, int64_t len) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < len) grad[i] -= 0.5f * (u[i] + v[i]);
}

// Cosine cost: x_i sqrt(1/2) / |x_i|, so that |x~_i - y~_j|^2 = 1 - cos(x_i, y_j). A zero
// point gives non-finite coordinates, which the coordinate check then reports.
__global__ void __launch_bounds__(256) normalize_kernel(const float* pts, int64_t count, int32_t d,
                                                        float* out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count) return;
  float s2 = 0.0f;
  for (int k = 0; k < d; ++k) s2 = fmaf(pts[i * d + k], pts[i * d + k], s2);
  const float sc = 0.70710678118654752f / sqrtf(s2);
  for (int k = 0; k < d; ++k) out[i * d + k] = pts[i * d + k] * sc;
}

// Cosine cost: the gradient with respect to x from the one with respect to
// x~ = sqrt(1/2) x / |x|: multiply by the Jacobian sqrt(1/2) (I - u u^T) / |x|, u = x / |x|.
__global__ void __launch_bounds__(256) cosine_grad_kernel(const float* pts, int64_t count, int32_t d,
                                                          float* grad) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count) return;
  float s2 = 0.0f, ug = 0.0f;
  for (int k = 0; k < d; ++k) s2 = fmaf(pts[i * d + k], pts[i * d + k], s2);
  const float inv = 1.0f / sqrtf(s2);
  for (int k = 0; k < d; ++k) ug = fmaf(pts[i * d + k] * inv, grad[i * d + k], ug);
  const float sc = 0.70710678118654752f * inv;
  for (int k = 0; k < d; ++k) grad[i * d + k] = sc * (grad[i * d + k] - pts[i * d + k] * inv * ug);
}

// Symmetric schedule: install the deferred biases of a cloud into its packed keys and
// record the smallest change (for the screening history bound of the next pass).
template <int D>
__global__ void __launch_bounds__(256) apply_bias_kernel(float* keys, const float* defer_h,
                                                         int64_t count, int* dmin_out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  float delta = INFINITY;
  if (i < count) {
    const int64_t slot = key_slot<D>(i, D);
    const float hn = defer_h[i];
    delta = hn - keys[slot];
    keys[slot] = hn;
  }
  reduce_dmin(delta, dmin_out);
}

// Potential stop check: the largest |v - prev| over a vector, then prev <- v. The maximum
// is kept as the bits of a non-negative float (ordered like unsigned ints).
__global__ void __launch_bounds__(256) pot_change_kernel(const float* v, float* prev, int64_t count,
                                                         unsigned* max_bits) {
  float mx = 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float x = v[i];
    mx = fmaxf(mx, fabsf(x - prev[i]));
    prev[i] = x;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) atomicMax(max_bits, __float_as_uint(mx));
}

__global__ void residual_finish_kernel(const double* row_acc, const double* col_acc, double* out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    out[0] = row_acc[0];
    out[1] = row_acc[1];
    out[2] = col_acc[0];
    out[3] = col_acc[1];
  }
}

// ---- error-path checks -------------------------------------------------------------------

// ORs `bits` into a call's error word from the device, where a kernel whose bounded wait
// expired would have set it (fault injection for the error path; no wait is involved).
__global__ void or_error_word_kernel(unsigned* err, unsigned bits) {
  if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(err, bits);
}

// Self-check of the bounded mbarrier wait every pass kernel uses: one thread waits for the
// first phase of a barrier that nothing arrives at (no copy or MMA is in flight), gives up
// after limit_ns and sets kErrTimeout in the error word, as a pass kernel would.
__global__ void bounded_wait_check_kernel(unsigned* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait_bounded(&bar, 0, limit_ns)) atomicOr(err, kErrTimeout);
}

}  // namespace fs
