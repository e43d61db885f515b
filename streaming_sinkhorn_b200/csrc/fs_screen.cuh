// fs_screen.cuh -- block screening of a streaming pass on spatially sorted clouds, and the
// balanced unit plan that the screened pass runs on.
//
// The screening bound. For a row i of a pass, every term is 2^z_ij with
// z_ij = H_j - kappa |x_i - y_j|^2 (log2 units). For a row block (the R*NT rows of one CTA)
// with bounding box B and a key tile T with box B_T and largest bias Hmax_T,
//   z_ij <= Hmax_T - kappa dist(B, B_T)^2 =: ub(T)          for all i in the block, j in T.
// A lower bound mlb_i on each row's largest exponent max_j z_ij comes from
//   (a) an anchor tile: max over the anchor's keys of the computed z_ij is a value the row
//       reaches (the anchor is the tile with the largest ub);
//   (b) history (potential passes after the first two): the largest term of a sum of m terms
//       is at least the sum over m, and every bias moved by at least dmin since the row's
//       previous pass, so max_j z_ij >= LSE2_prev_i + dmin - log2(m).
// A tile with ub(T) < min_i mlb_i - margin is skipped. Each of its terms is below
// 2^-margin times its row's largest term, so with margin = kSkipBits + log2(m) the whole
// omitted part of a row's sum is below 2^-kSkipBits of that sum (the largest term is at
// most the sum). With kSkipBits = 32 this is under the rounding of the fp32 sums. The
// anchor is always kept, so every row block has work.
//
// The plan. The kept tiles of a row block are cut into units of at most C tiles, with C
// the smallest count that keeps the number of units under a budget sized from the SM
// count; the pass then runs one CTA per unit. Row blocks with many kept tiles (dense
// clusters, block boxes across a jump of the space-filling curve) become several units,
// so no CTA carries far more work than the others, and a row block's units are merged by
// the second-level LSE of combine_kernel.
#pragma once

#include "fs_kernels.cuh"

namespace fs {

// One warp (one CTA) per row block of 32 R rows: the bit mask of kept key tiles and its
// population count. Tiles are tested through their super-tiles first: a super-tile's box
// contains its tiles' boxes and its bias maximum bounds theirs, so its upper bound bounds
// theirs, and a rejected super-tile rejects all of its tiles.
template <int D, int R>
__global__ void __launch_bounds__(32) screen_kernel(const PassParams P, unsigned* kmask,
                                                    int* kcount) {
  constexpr int KP = key_pair_floats(D);
  constexpr int RB = R * 32;
  constexpr int TP = kScreenTile / 2;  // key pairs per tile
  __shared__ __align__(16) float anchor_tile[TP * KP];
  const int lane = threadIdx.x;
  const int64_t b = blockIdx.x;
  const int64_t row0 = b * RB;
  const int T = P.key_tiles, S = P.key_supers;

  // rows of the block and their box (every lane ends with the block's box)
  float x[R][D];
  bool valid[R];
  float lo[D], hi[D];
#pragma unroll
  for (int k = 0; k < D; ++k) {
    lo[k] = INFINITY;
    hi[k] = -INFINITY;
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t i = row0 + r * 32 + lane;
    valid[r] = i < P.n_rows;
#pragma unroll
    for (int k = 0; k < D; ++k) {
      x[r][k] = valid[r] ? P.qkeys[key_slot<D>(i, k)] : 0.0f;
      if (valid[r]) {
        lo[k] = fminf(lo[k], x[r][k]);
        hi[k] = fmaxf(hi[k], x[r][k]);
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
  // upper bound of the exponents of entry idx of a component-major summary (stride n)
  auto ub_of = [&](const float* box, const float* hm, int n, int idx) -> float {
    float d2 = 0.0f;
#pragma unroll
    for (int k = 0; k < D; ++k) {
      const float gap = fmaxf(fmaxf(box[k * n + idx] - hi[k], lo[k] - box[(D + k) * n + idx]), 0.0f);
      d2 = fmaf(gap, gap, d2);
    }
    return hm[idx] - P.kappa_f * d2;
  };
  // warp argmax of (ub, -index): key = ordered ub << 32 | ~index
  auto best_of = [&](float ub, int idx, bool ok) -> unsigned long long {
    unsigned long long key =
        ok ? (static_cast<unsigned long long>(static_cast<unsigned>(float_ord(ub)) ^ 0x80000000u) << 32) |
                 static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<unsigned>(idx))
           : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
      key = key > other ? key : other;
    }
    return key;
  };

  // anchor: the tile with the largest upper bound (ties to the lower index), found through
  // the super-tiles: the best tile of the best super-tile gives a bound L, and only
  // super-tiles whose own bound exceeds L can hold a better tile.
  unsigned long long best = 0ull;
  for (int s0 = 0; s0 < S; s0 += 32) {
    const int sidx = s0 + lane;
    const unsigned long long k = best_of(sidx < S ? ub_of(P.key_sbox, P.key_shmax, S, sidx) : 0.0f,
                                         sidx, sidx < S);
    best = best > k ? best : k;
  }
  const int sstar = static_cast<int>(0xFFFFFFFFu - static_cast<unsigned>(best & 0xFFFFFFFFull));
  {
    const int t = sstar * kSuper + lane;
    const bool ok = lane < kSuper && t < T;
    best = best_of(ok ? ub_of(P.key_box, P.key_hmax, T, t) : 0.0f, t, ok);
  }
  for (int s0 = 0; s0 < S; s0 += 32) {
    const int sidx = s0 + lane;
    const float lbest = ord_float(static_cast<int>(static_cast<unsigned>(best >> 32) ^ 0x80000000u));
    unsigned sbits = __ballot_sync(
        0xffffffffu, sidx < S && sidx != sstar && ub_of(P.key_sbox, P.key_shmax, S, sidx) >= lbest);
    while (sbits) {
      const int sl = __ffs(sbits) - 1;
      sbits &= sbits - 1u;
      const int t = (s0 + sl) * kSuper + lane;
      const bool ok = lane < kSuper && t < T;
      const unsigned long long k = best_of(ok ? ub_of(P.key_box, P.key_hmax, T, t) : 0.0f, t, ok);
      best = best > k ? best : k;
    }
  }
  const int anchor = static_cast<int>(0xFFFFFFFFu - static_cast<unsigned>(best & 0xFFFFFFFFull));

  // the anchor's keys, then each row's largest exponent over them (packed, direct form)
  {
    const float4* src = reinterpret_cast<const float4*>(P.keys + static_cast<int64_t>(anchor) * TP * KP);
    float4* dst = reinterpret_cast<float4*>(anchor_tile);
    for (int q = lane; q < TP * KP / 4; q += 32) dst[q] = src[q];
  }
  __syncwarp();
  u64 xp[R][D];
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int k = 0; k < D; ++k) xp[r][k] = pk(x[r][k], x[r][k]);
  }
  const u64 nkappa = pk(-P.kappa_f, -P.kappa_f);
  float zmax[R];
#pragma unroll
  for (int r = 0; r < R; ++r) zmax[r] = -INFINITY;
#pragma unroll 4
  for (int p = 0; p < TP; ++p) {
    u64 comp[KP / 2];
    load_pair<KP>(anchor_tile, p, comp);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      u64 acc = pk(0.0f, 0.0f);
#pragma unroll
      for (int k = 0; k < D; ++k) {
        const u64 dk = sub2(xp[r][k], comp[k]);
        acc = fma2(dk, dk, acc);
      }
      float z0, z1;
      upk(fma2(nkappa, acc, comp[D]), z0, z1);
      zmax[r] = max3(zmax[r], z0, z1);
    }
  }
  const bool history = P.lse_prev && P.key_dmin;
  const float dmin = history ? ord_float(*P.key_dmin) : 0.0f;
  float mlb = INFINITY;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (!valid[r]) continue;
    const int64_t i = row0 + r * 32 + lane;
    float v = zmax[r];
    if (history) v = fmaxf(v, P.lse_prev[i] + dmin - P.log2_keys);
    if (P.row_mlb) P.row_mlb[i] = v;
    mlb = fminf(mlb, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mlb = fminf(mlb, __shfl_xor_sync(0xffffffffu, mlb, o));
  const float thr = mlb - P.skip_margin;

  // the mask, 32 super-tiles (8 mask words) per round; lane j < 8 assembles word j
  unsigned* mrow = kmask + b * P.mask_words;
  int cnt = 0;
  for (int s0 = 0; s0 < S; s0 += 32) {
    const int sidx = s0 + lane;
    const bool keep_s =
        sidx < S && (sidx == anchor / kSuper || ub_of(P.key_sbox, P.key_shmax, S, sidx) >= thr);
    unsigned sbits = __ballot_sync(0xffffffffu, keep_s);
    unsigned word = 0u;
    while (sbits) {
      const int sl = __ffs(sbits) - 1;
      sbits &= sbits - 1u;
      const int t = (s0 + sl) * kSuper + lane;
      const bool keep_t =
          lane < kSuper && t < T && (t == anchor || ub_of(P.key_box, P.key_hmax, T, t) >= thr);
      const unsigned pat = __ballot_sync(0xffffffffu, keep_t) & 0xFFu;
      if (lane == sl / 4) word |= pat << ((sl % 4) * kSuper);
    }
    const int w = s0 / 4 + lane;
    if (lane < 8 && w < P.mask_words) {
      mrow[w] = word;
      cnt += __popc(word);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) kcount[b] = cnt;
}

// One CTA of 1024 threads: C = max(1, ceil(K / budget)) for K kept tiles in all; each row
// block's kept tiles in units of C (floor(kept / C) full units and one shorter tail unit when
// C does not divide kept); the prefix of units per block (partial slots and unit counts for
// the merge); and the launch order: every full unit first, in block order, then the tails,
// so that the last CTAs the hardware schedules are the shortest ones. Also K itself and the
// evaluated-pair count (kept tiles x 256 keys x rows per block).
__global__ void __launch_bounds__(1024) plan_units_kernel(const int* kcount, int rb,
                                                          long long budget, int rb_rows,
                                                          int* unit_start, int* unit_rb,
                                                          int* unit_j, int* qscal,
                                                          long long* kept_out,
                                                          unsigned long long* evaluated) {
  __shared__ long long s_part[32];
  __shared__ int s_scan[3][32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  // thread t owns row blocks [t * per, (t + 1) * per)
  const int per = (rb + 1023) / 1024;
  const int b0 = min(rb, tid * per), b1 = min(rb, b0 + per);
  long long k = 0;
  for (int b = b0; b < b1; ++b) k += kcount[b];
  long long kw = k;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) kw += __shfl_xor_sync(0xffffffffu, kw, o);
  if (lane == 0) s_part[wid] = kw;
  __syncthreads();
  long long total = 0;
  for (int q = 0; q < 32; ++q) total += s_part[q];
  const int C = static_cast<int>(total > budget ? (total + budget - 1) / budget : 1);
  // per thread: units, full units and tail units of its blocks
  int v[3] = {0, 0, 0};
  for (int b = b0; b < b1; ++b) {
    const int kc = kcount[b];
    v[1] += kc / C;
    v[2] += kc % C ? 1 : 0;
  }
  v[0] = v[1] + v[2];
  int incl[3], excl[3], all[3];
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    incl[q] = v[q];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl[q], o);
      if (lane >= o) incl[q] += t;
    }
    if (lane == 31) s_scan[q][wid] = incl[q];
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    int wbase = 0;
    all[q] = 0;
    for (int w = 0; w < 32; ++w) {
      if (w < wid) wbase += s_scan[q][w];
      all[q] += s_scan[q][w];
    }
    excl[q] = wbase + incl[q] - v[q];
  }
  int start = excl[0], full = excl[1], tail = all[1] + excl[2];
  for (int b = b0; b < b1; ++b) {
    const int kc = kcount[b];
    const int nf = kc / C;
    unit_start[b] = start;
    start += nf + (kc % C ? 1 : 0);
    for (int j = 0; j < nf; ++j) {
      unit_rb[full + j] = b;
      unit_j[full + j] = j;
    }
    full += nf;
    if (kc % C) {
      unit_rb[tail] = b;
      unit_j[tail] = nf;
      ++tail;
    }
  }
  if (tid == 1023) {
    unit_start[rb] = start;
    qscal[0] = C;
    qscal[1] = start;
    *kept_out = total;
    if (evaluated)
      atomicAdd(evaluated, static_cast<unsigned long long>(total) * kScreenTile * rb_rows);
  }
}

}  // namespace fs
