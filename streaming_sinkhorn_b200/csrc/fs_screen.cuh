// fs_screen.cuh -- block screening of a streaming pass on spatially sorted clouds, and the
// balanced unit plan that the screened pass runs on.
//
// The screening bound. For a row i of a pass, every term is 2^z_ij with
// z_ij = H_j - kappa |x_i - y_j|^2 (log2 units). For a row block (the R*NT rows of one CTA)
// with bounding box B and a key tile T with box B_T and largest bias Hmax_T,
//   z_ij <= Hmax_T - kappa dist(B, B_T)^2 =: ub(T)          for all i in the block, j in T.
// A lower bound mlb_i on each row's largest exponent max_j z_ij comes from
//   (a) anchor tiles: the max over an anchor's keys of the computed z_ij is a value the row
//       reaches. The anchors are the key tiles that hold the row block's stretch of the
//       Morton order both clouds share (the keys whose codes lie between the block's first
//       and last row codes, and one key on either side): they hold most rows' nearest keys,
//       so the bound is close to each row's true maximum, at most kMortonAnchors of them.
//       A screen may record, per row, the key that gave this maximum; a later screen of the
//       same call evaluates z_ij at that key alone (only the biases H changed in between,
//       and any key's exponent is a value the row reaches);
//   (b) history (potential passes after the first two): the largest term of a sum of m terms
//       is at least the sum over m, and every bias moved by at least dmin since the row's
//       previous pass, so max_j z_ij >= LSE2_prev_i + dmin - log2(m).
// A tile with ub(T) < min_i mlb_i - margin is skipped, and so is a tile for which every row
// i of the block has ub_i(T) = Hmax_T - kappa dist(x_i, B_T)^2 < mlb_i - margin (the same
// bound for the row alone). Each of its terms is below
// 2^-margin times its row's largest term, so with margin = kSkipBits + log2(m) the whole
// omitted part of a row's sum is below 2^-kSkipBits of that sum (the largest term is at
// most the sum). With kSkipBits = 24, the fp32 unit roundoff, the omitted mass is at most
// one rounding of the row's sum (the fp32 accumulation itself errs by more). The first
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

// Super-tile bounds a screening warp keeps in shared memory (4 KiB); beyond this many
// super-tiles (2^21 keys) it recomputes them where they are used.
constexpr int kSupCache = 1024;
// Anchor tiles a screening warp evaluates at most (spread over the block's Morton stretch).
constexpr int kMortonAnchors = 4;

// One warp (one CTA) per row block of 32 R rows: the bit mask of kept key tiles and its
// population count. Tiles are tested through their super-tiles first: a super-tile's box
// contains its tiles' boxes and its bias maximum bounds theirs, so its upper bound bounds
// theirs, and a rejected super-tile rejects all of its tiles.
template <int D, int R>
__global__ void __launch_bounds__(32) screen_kernel(const PassParams P, unsigned* kmask,
                                                    int* kcount) {
  static_assert(R == 2, "the per-row tile test packs a lane's two rows");
  constexpr int KP = key_pair_floats(D);
  constexpr int RB = R * 32;
  constexpr int TP = kScreenTile / 2;  // key pairs per tile
  __shared__ __align__(16) float anchor_tile[TP * KP];
  extern __shared__ float s_sub[];  // kSupCache bounds at most (dynamic size)
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
  // Super-tile bounds, kept in shared memory when they fit (every lane reads back only the
  // entries it wrote, so no barrier is needed); otherwise recomputed where used.
  const bool cached = S <= kSupCache;
  auto sub_ub = [&](int sidx) -> float {
    return cached ? s_sub[sidx] : ub_of(P.key_sbox, P.key_shmax, S, sidx);
  };

  if (cached)
    for (int sidx = lane; sidx < S; sidx += 32) s_sub[sidx] = ub_of(P.key_sbox, P.key_shmax, S, sidx);

  // Each row's largest exponent over the keys of a few tiles is a value the row reaches.
  // A tile's keys are taken about the block's centre c (y' = y - c, H' = H - kappa |y'|^2):
  // z = H' - kappa |x'|^2 + 2 kappa x'.y' (packed).
  u64 cpk[D];
#pragma unroll
  for (int k = 0; k < D; ++k) {
    const float c = lo[k] <= hi[k] ? 0.5f * (lo[k] + hi[k]) : 0.0f;
    cpk[k] = pk(c, c);
  }
  const u64 nkappa = pk(-P.kappa_f, -P.kappa_f);
  u64 xp[R][D], mk[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float s2 = 0.0f;
#pragma unroll
    for (int k = 0; k < D; ++k) {
      float cc, cd;
      upk(cpk[k], cc, cd);
      const float xs = x[r][k] - cc;
      s2 = fmaf(xs, xs, s2);
      const float x2 = 2.0f * P.kappa_f * xs;
      xp[r][k] = pk(x2, x2);
    }
    const float q = -P.kappa_f * s2;
    mk[r] = pk(q, q);
  }
  float zmax[R];
  int zarg[R];  // anchor_mode 1: the key (sorted order) of each row's largest anchor exponent
#pragma unroll
  for (int r = 0; r < R; ++r) {
    zmax[r] = -INFINITY;
    zarg[r] = -1;
  }
  const bool record = P.anchor_key && P.anchor_mode == 1;
  auto eval_tile = [&](int t) {
    __syncwarp();  // every lane is done with the previous tile
    const float* src = P.keys + static_cast<int64_t>(t) * TP * KP;
    for (int p = lane; p < TP; p += 32) {
      u64 comp[KP / 2];
      load_pair<KP>(src, p, comp);
      u64 s2 = pk(0.0f, 0.0f);
#pragma unroll
      for (int k = 0; k < D; ++k) {
        comp[k] = sub2(comp[k], cpk[k]);
        s2 = fma2(comp[k], comp[k], s2);
      }
      comp[D] = fma2(nkappa, s2, comp[D]);
      ulonglong2* pv = reinterpret_cast<ulonglong2*>(anchor_tile + p * KP);
#pragma unroll
      for (int v = 0; v < KP / 4; ++v) pv[v] = make_ulonglong2(comp[2 * v], comp[2 * v + 1]);
    }
    __syncwarp();
#pragma unroll 4
    for (int p = 0; p < TP; ++p) {
      u64 comp[KP / 2];
      load_pair<KP>(anchor_tile, p, comp);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        u64 acc = add2(comp[D], mk[r]);
#pragma unroll
        for (int k = 0; k < D; ++k) acc = fma2(xp[r][k], comp[k], acc);
        float z0, z1;
        upk(acc, z0, z1);
        if (record) {
          const int key0 = t * kScreenTile + 2 * p;
          if (z0 > zmax[r]) {
            zmax[r] = z0;
            zarg[r] = key0;
          }
          if (z1 > zmax[r]) {
            zmax[r] = z1;
            zarg[r] = key0 + 1;
          }
        } else {
          zmax[r] = max3(zmax[r], z0, z1);
        }
      }
    }
  };

  // The anchors: the key tiles that hold the block's stretch of the shared Morton order
  // (from one key before the block's first row code to one key after its last), at most
  // kMortonAnchors of them, spread over the stretch. Without codes no tile is evaluated,
  // every bound stays -inf and every tile is kept.
  int anchor = -1;
  if (P.anchor_key && P.anchor_mode == 2) {
    // the recorded key of each row: its exponent now (direct difference)
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!valid[r]) continue;
      // a recorded key index; clamped so that even a stale one stays inside the keys
      const int j = min(max(P.anchor_key[row0 + r * 32 + lane], 0),
                        static_cast<int>(P.key_count) - 1);
      float d2 = 0.0f;
#pragma unroll
      for (int k = 0; k < D; ++k) {
        const float dk = x[r][k] - P.keys[key_slot<D>(j, k)];
        d2 = fmaf(dk, dk, d2);
      }
      zmax[r] = P.keys[key_slot<D>(j, D)] - P.kappa_f * d2;
    }
    // the tile of the first row's key is always kept, so the block has work
    anchor = min(max(P.anchor_key[row0], 0), static_cast<int>(P.key_count) - 1) / kScreenTile;
  } else if (P.key_codes) {
    const int64_t nk = P.key_count;
    // first position in the sorted key codes whose code is >= target (warp-wide search)
    auto lower_bound = [&](uint64_t target) -> int64_t {
      int64_t lo_p = 0, hi_p = nk;
      while (hi_p - lo_p > 32) {
        const int64_t q = lo_p + (static_cast<int64_t>(lane) + 1) * (hi_p - lo_p) / 33;
        const unsigned below = __ballot_sync(0xffffffffu, P.key_codes[q] < target);
        const int c = __popc(below);
        const int64_t nlo = c == 0 ? lo_p : __shfl_sync(0xffffffffu, q, c - 1) + 1;
        const int64_t nhi = c == 32 ? hi_p : __shfl_sync(0xffffffffu, q, c & 31);
        lo_p = nlo;
        hi_p = nhi;
      }
      const int64_t q = lo_p + lane;
      return lo_p + __popc(__ballot_sync(0xffffffffu, q < hi_p && P.key_codes[q] < target));
    };
    const int64_t last = (row0 + RB < P.n_rows ? row0 + RB : P.n_rows) - 1;
    const int64_t p0 = lower_bound(P.row_codes[row0]);
    const int64_t p1 = lower_bound(static_cast<uint64_t>(P.row_codes[last]) + 1u);
    const int64_t q0 = p0 > 0 ? p0 - 1 : 0;
    const int64_t q1 = p1 < nk - 1 ? p1 : nk - 1;
    const int t0 = static_cast<int>(q0 / kScreenTile), t1 = static_cast<int>(q1 / kScreenTile);
    const int span = t1 - t0 + 1;
    const int na = span < kMortonAnchors ? span : kMortonAnchors;
    for (int e = 0; e < na; ++e) {
      const int t = na == span ? t0 + e : t0 + static_cast<int>(static_cast<int64_t>(e) * (span - 1) / (na - 1));
      if (e == 0) anchor = t;
      eval_tile(t);
    }
  }
  if (record) {
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (valid[r] && zarg[r] >= 0) P.anchor_key[row0 + r * 32 + lane] = zarg[r];
  }
  const bool history = P.lse_prev && P.key_dmin;
  const float dmin = history ? ord_float(*P.key_dmin) : 0.0f;
  float mlb = INFINITY;
  float rthr[R];  // each row's own threshold (+inf for rows past the end)
#pragma unroll
  for (int r = 0; r < R; ++r) {
    rthr[r] = INFINITY;
    if (!valid[r]) continue;
    const int64_t i = row0 + r * 32 + lane;
    float v = zmax[r];
    if (history) v = fmaxf(v, P.lse_prev[i] + dmin - P.log2_keys);
    mlb = fminf(mlb, v);
    rthr[r] = v - P.skip_margin;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mlb = fminf(mlb, __shfl_xor_sync(0xffffffffu, mlb, o));
  const float thr = mlb - P.skip_margin;
  // each row's own threshold, for the pass's skip of 16-point groups inside kept tiles
  if (P.row_thr) {
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (valid[r]) P.row_thr[row0 + r * 32 + lane] = rthr[r];
  }

  // The mask, 32 super-tiles (8 mask words) per round; lane j < 8 assembles word j. A tile
  // is tested against the block's box and smallest bound, then each tile that passes row by
  // row: it stays only if some row i has Hmax_t - kappa dist(x_i, B_t)^2 >= its own bound
  // - margin. A block whose box spans two clusters, or that holds a row far below the
  // others, keeps many tiles under the block test; the per-row test removes most of them.
  // A lane tests its two rows at once in packed arithmetic.
  u64 xr[D];
#pragma unroll
  for (int k = 0; k < D; ++k) xr[k] = pk(x[0][k], x[1][k]);
  unsigned* mrow = kmask + b * P.mask_words;
  int cnt = 0;
  for (int s0 = 0; s0 < S; s0 += 32) {
    const int sidx = s0 + lane;
    const bool keep_s = sidx < S && (sidx == anchor / kSuper || sub_ub(sidx) >= thr);
    unsigned sbits = __ballot_sync(0xffffffffu, keep_s);
    unsigned word = 0u;
    // Up to four kept super-tiles at a time: lane l loads tile l % 8 of the (l / 8)-th one
    // (box and Hmax), so one round trip to L2 serves 32 tiles; the per-row tests below take
    // them by shuffles.
    while (sbits) {
      int sl[4];
      int nsup = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        sl[q] = sbits ? __ffs(sbits) - 1 : -1;
        if (sbits) {
          sbits &= sbits - 1u;
          ++nsup;
        }
      }
      const int q = lane / kSuper;
      const int myq_sl = q == 0 ? sl[0] : (q == 1 ? sl[1] : (q == 2 ? sl[2] : sl[3]));
      const int t = myq_sl >= 0 ? (s0 + myq_sl) * kSuper + lane % kSuper : -1;
      const bool okl = q < nsup && t >= 0 && t < T;
      float blo[D], bhi[D];
      float d2b = 0.0f;
#pragma unroll
      for (int k = 0; k < D; ++k) {
        blo[k] = okl ? P.key_box[k * T + t] : 0.0f;
        bhi[k] = okl ? P.key_box[(D + k) * T + t] : 0.0f;
        const float gap = fmaxf(fmaxf(blo[k] - hi[k], lo[k] - bhi[k]), 0.0f);
        d2b = fmaf(gap, gap, d2b);
      }
      const float thm = okl ? P.key_hmax[t] : -INFINITY;
      const bool keep_t = okl && (t == anchor || thm - P.kappa_f * d2b >= thr);
      unsigned pat = __ballot_sync(0xffffffffu, keep_t);
      unsigned test = pat;
      while (test) {
        const int tl = __ffs(test) - 1;
        test &= test - 1u;
        const int ttile = __shfl_sync(0xffffffffu, t, tl);
        if (ttile == anchor) continue;
        u64 d2 = pk(0.0f, 0.0f);
#pragma unroll
        for (int k = 0; k < D; ++k) {
          const float lk = __shfl_sync(0xffffffffu, blo[k], tl);
          const float hk = __shfl_sync(0xffffffffu, bhi[k], tl);
          float a0, a1, c0, c1;
          upk(sub2(pk(lk, lk), xr[k]), a0, a1);
          upk(sub2(xr[k], pk(hk, hk)), c0, c1);
          const u64 gap = pk(max3(a0, c0, 0.0f), max3(a1, c1, 0.0f));
          d2 = fma2(gap, gap, d2);
        }
        float e0, e1;
        upk(d2, e0, e1);
        const float hm = __shfl_sync(0xffffffffu, thm, tl);
        const bool need = hm - P.kappa_f * e0 >= rthr[0] || hm - P.kappa_f * e1 >= rthr[1];
        if (!__any_sync(0xffffffffu, need)) pat &= ~(1u << tl);
      }
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        if (qq < nsup && lane == sl[qq] / 4)
          word |= ((pat >> (qq * kSuper)) & 0xFFu) << ((sl[qq] % 4) * kSuper);
      }
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
  __shared__ long long s_kept[32];
  __shared__ int s_cnt[3][32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  // warp w owns the run of row blocks [w0, w1), read 32 consecutive blocks at a time
  const int per_w = (rb + 31) / 32;
  const int w0 = min(rb, wid * per_w), w1 = min(rb, w0 + per_w);
  long long k = 0;
#pragma unroll 4
  for (int b = w0 + lane; b < w1; b += 32) k += kcount[b];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
  if (lane == 0) s_kept[wid] = k;
  __syncthreads();
  long long total = 0;
  for (int q = 0; q < 32; ++q) total += s_kept[q];
  const int C = static_cast<int>(total > budget ? (total + budget - 1) / budget : 1);
  // per warp: units, full units and tail units of its run
  int v[3] = {0, 0, 0};
#pragma unroll 4
  for (int b = w0 + lane; b < w1; b += 32) {
    const int kc = kcount[b];
    const int nf = kc / C;
    v[1] += nf;
    v[2] += kc - nf * C ? 1 : 0;
  }
  v[0] = v[1] + v[2];
#pragma unroll
  for (int q = 0; q < 3; ++q) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[q] += __shfl_xor_sync(0xffffffffu, v[q], o);
    if (lane == 0) s_cnt[q][wid] = v[q];
  }
  __syncthreads();
  // exclusive prefix of the warps' counts (lane l holds warp l's) and the totals
  int base[3], all[3];
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    const int own = s_cnt[q][lane];
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    base[q] = __shfl_sync(0xffffffffu, incl - own, wid);
    all[q] = __shfl_sync(0xffffffffu, incl, 31);
  }
  // the run's units in rounds of 32 blocks: a scan within the round gives each block its
  // first unit (merge order), its full units' slots and its tail's slot (launch order)
  int start = base[0], full = base[1], tail = all[1] + base[2];
  for (int r0 = w0; r0 < w1; r0 += 32) {
    const int b = r0 + lane;
    const int kc = b < w1 ? kcount[b] : 0;
    const int nf = kc / C;
    const int tl = kc - nf * C ? 1 : 0;
    int iu = nf + tl, ifl = nf, itl = tl;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, iu, o);
      const int f = __shfl_up_sync(0xffffffffu, ifl, o);
      const int t = __shfl_up_sync(0xffffffffu, itl, o);
      if (lane >= o) {
        iu += a;
        ifl += f;
        itl += t;
      }
    }
    if (b < w1) {
      unit_start[b] = start + iu - (nf + tl);
      const int f0 = full + ifl - nf;
      for (int j = 0; j < nf; ++j) {
        unit_rb[f0 + j] = b;
        unit_j[f0 + j] = j;
      }
      if (tl) {
        unit_rb[tail + itl - 1] = b;
        unit_j[tail + itl - 1] = nf;
      }
    }
    start += __shfl_sync(0xffffffffu, iu, 31);
    full += __shfl_sync(0xffffffffu, ifl, 31);
    tail += __shfl_sync(0xffffffffu, itl, 31);
  }
  if (tid == 0) {
    unit_start[rb] = all[0];
    qscal[0] = C;
    qscal[1] = all[0];
    *kept_out = total;
    if (evaluated)
      atomicAdd(evaluated, static_cast<unsigned long long>(total) * kScreenTile * rb_rows);
  }
}

}  // namespace fs
