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

// One CTA per row block: the bit mask of kept key tiles and its population count.
template <int D, int R, int NT>
__global__ void __launch_bounds__(NT) screen_kernel(const PassParams P, unsigned* kmask,
                                                    int* kcount) {
  constexpr int KP = key_pair_floats(D);
  constexpr int RB = R * NT;
  constexpr int TP = kScreenTile / 2;  // key pairs per tile
  extern __shared__ __align__(16) float anchor_tile[];  // TP * KP floats
  __shared__ int s_box[2 * D];
  __shared__ int s_mlb, s_cnt;
  __shared__ unsigned long long s_best;
  const int tid = threadIdx.x;
  const int64_t b = blockIdx.x;
  const int64_t row0 = b * RB;
  const int n_tiles = static_cast<int>(P.key_pairs / TP);
  if (tid < D) {
    s_box[tid] = 0x7FFFFFFF;
    s_box[D + tid] = static_cast<int>(0x80000000u);
  }
  if (tid == 0) {
    s_mlb = 0x7FFFFFFF;
    s_cnt = 0;
    s_best = 0ull;
  }
  __syncthreads();

  // rows of the block and their box
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
    const int64_t i = row0 + r * NT + tid;
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
  if ((tid & 31) == 0) {
#pragma unroll
    for (int k = 0; k < D; ++k) {
      atomicMin(&s_box[k], float_ord(lo[k]));
      atomicMax(&s_box[D + k], float_ord(hi[k]));
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < D; ++k) {
    lo[k] = ord_float(s_box[k]);
    hi[k] = ord_float(s_box[D + k]);
  }
  auto tile_ub = [&](int tt) -> float {
    const float* bx = P.key_box + static_cast<int64_t>(tt) * 2 * D;
    float d2 = 0.0f;
#pragma unroll
    for (int k = 0; k < D; ++k) {
      const float gap = fmaxf(fmaxf(bx[k] - hi[k], lo[k] - bx[D + k]), 0.0f);
      d2 = fmaf(gap, gap, d2);
    }
    return P.key_hmax[tt] - P.kappa_f * d2;
  };

  // anchor: the largest upper bound, ties to the lower tile index
  unsigned long long best = 0ull;
  for (int tt = tid; tt < n_tiles; tt += NT) {
    const unsigned ub = static_cast<unsigned>(float_ord(tile_ub(tt))) ^ 0x80000000u;
    const unsigned long long key = (static_cast<unsigned long long>(ub) << 32) |
                                   static_cast<unsigned long long>(0xFFFFFFFFu - tt);
    best = best > key ? best : key;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
    best = best > other ? best : other;
  }
  if ((tid & 31) == 0) atomicMax(&s_best, best);
  __syncthreads();
  const int anchor = static_cast<int>(0xFFFFFFFFu - static_cast<unsigned>(s_best & 0xFFFFFFFFull));

  // the anchor's keys, then each row's largest exponent over them
  {
    const float4* src = reinterpret_cast<const float4*>(P.keys + static_cast<int64_t>(anchor) * TP * KP);
    float4* dst = reinterpret_cast<float4*>(anchor_tile);
    for (int q = tid; q < TP * KP / 4; q += NT) dst[q] = src[q];
  }
  __syncthreads();
  float zmax[R];
#pragma unroll
  for (int r = 0; r < R; ++r) zmax[r] = -INFINITY;
  for (int p = 0; p < TP; ++p) {
    const float* kp = anchor_tile + p * KP;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float h = kp[2 * D + e];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float d2 = 0.0f;
#pragma unroll
        for (int k = 0; k < D; ++k) {
          const float dk = x[r][k] - kp[2 * k + e];
          d2 = fmaf(dk, dk, d2);
        }
        zmax[r] = fmaxf(zmax[r], fmaf(-P.kappa_f, d2, h));
      }
    }
  }
  const bool history = P.lse_prev && P.key_dmin;
  const float dmin = history ? ord_float(*P.key_dmin) : 0.0f;
  float mlb = INFINITY;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (!valid[r]) continue;
    float v = zmax[r];
    if (history) v = fmaxf(v, P.lse_prev[row0 + r * NT + tid] + dmin - P.log2_keys);
    mlb = fminf(mlb, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mlb = fminf(mlb, __shfl_xor_sync(0xffffffffu, mlb, o));
  if ((tid & 31) == 0) atomicMin(&s_mlb, float_ord(mlb));
  __syncthreads();
  const float thr = ord_float(s_mlb) - P.skip_margin;

  // the mask: one warp writes 32 consecutive tiles per word
  unsigned* mrow = kmask + b * P.mask_words;
  int cnt = 0;
  for (int base = 0; base < n_tiles; base += NT) {
    const int tt = base + tid;
    const bool keep = tt < n_tiles && (tt == anchor || tile_ub(tt) >= thr);
    const unsigned word = __ballot_sync(0xffffffffu, keep);
    const int w = (base + (tid & ~31)) >> 5;
    if ((tid & 31) == 0 && w < P.mask_words) {
      mrow[w] = word;
      cnt += __popc(word);
    }
  }
  if ((tid & 31) == 0) atomicAdd(&s_cnt, cnt);
  __syncthreads();
  if (tid == 0) kcount[b] = s_cnt;
}

// One CTA of 1024 threads: C = max(1, ceil(K / budget)) for K kept tiles in all, the units
// of each row block (ceil(kept / C)), their prefix, the row block of every unit, K itself
// and the evaluated-pair count (kept tiles x 256 keys x rows per block).
__global__ void __launch_bounds__(1024) plan_units_kernel(const int* kcount, int rb,
                                                          long long budget, int rb_rows,
                                                          int* unit_start, int* unit_rb,
                                                          int* qscal, long long* kept_out,
                                                          unsigned long long* evaluated) {
  __shared__ long long s_part[32];
  __shared__ int s_scan[32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  long long k = 0;
  for (int b = tid; b < rb; b += 1024) k += kcount[b];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
  if (lane == 0) s_part[wid] = k;
  __syncthreads();
  long long total = 0;
  for (int q = 0; q < 32; ++q) total += s_part[q];
  const long long C = total > budget ? (total + budget - 1) / budget : 1;
  int carry = 0;
  for (int base = 0; base < rb; base += 1024) {
    const int b = base + tid;
    const int nu = b < rb ? static_cast<int>((kcount[b] + C - 1) / C) : 0;
    int incl = nu;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    __syncthreads();  // s_scan free from the previous round
    if (lane == 31) s_scan[wid] = incl;
    __syncthreads();
    int wbase = 0;
    for (int q = 0; q < wid; ++q) wbase += s_scan[q];
    int all = 0;
    for (int q = 0; q < 32; ++q) all += s_scan[q];
    const int start = carry + wbase + incl - nu;
    if (b < rb) {
      unit_start[b] = start;
      for (int j = 0; j < nu; ++j) unit_rb[start + j] = b;
    }
    carry += all;
  }
  if (tid == 0) {
    unit_start[rb] = carry;
    qscal[0] = static_cast<int>(C);
    qscal[1] = carry;
    *kept_out = total;
    if (evaluated)
      atomicAdd(evaluated, static_cast<unsigned long long>(total) * kScreenTile * rb_rows);
  }
}

}  // namespace fs
