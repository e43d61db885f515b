// fs_sort.cuh -- spatial order of a point cloud and per-tile summaries for block screening.
//
// Points are put in Morton (Z-curve) order of their first three coordinates, quantised on
// the common bounding box of both clouds, so that each run of 256 consecutive points (one
// screening tile) is spatially compact. The order is a bitonic sort of unique 64-bit keys
// (Morton code << 32 | original index), so it is deterministic. For every tile the pass
// needs the coordinate bounding box and the largest key bias H over its points; with them
// a CTA can bound every score of a tile from above without touching its points (the
// block-sparse screening of the FlashSinkhorn 2 abstract, here with a bound that makes the
// omitted mass provably negligible rather than a tolerance).
#pragma once

#include <cstdint>
#include "fs_device.cuh"

namespace fs {

constexpr int kSortDims = 3;       // coordinates entering the Morton code
constexpr int kSortBlock = 1024;   // threads of the shared-memory bitonic kernels
constexpr int kSortSmem = 2 * kSortBlock;  // keys sorted per block in shared memory

// Order-preserving int image of a float, for atomicMin/atomicMax on floats.
__device__ __forceinline__ int float_ord(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__host__ __device__ __forceinline__ float ord_float(int i) {
  const int b = i >= 0 ? i : i ^ 0x7FFFFFFF;
  float f;
  memcpy(&f, &b, sizeof(float));
  return f;
}

// Bounding box of the first min(d, 3) coordinates: ordered ints in lo[3], hi[3].
__global__ void __launch_bounds__(256) bbox_kernel(const float* pts, int64_t count, int32_t d,
                                                   int* lo, int* hi) {
  const int k = blockIdx.y;
  float mn = INFINITY, mx = -INFINITY;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < count;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = pts[j * d + k];
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if ((threadIdx.x & 31) == 0) {
    atomicMin(&lo[k], float_ord(mn));
    atomicMax(&hi[k], float_ord(mx));
  }
}

__device__ __forceinline__ uint32_t spread_bits(uint32_t v, int dims) {
  if (dims == 3) {  // 10 bits -> every third bit of 30
    v &= 0x3FFu;
    v = (v | (v << 16)) & 0x030000FFu;
    v = (v | (v << 8)) & 0x0300F00Fu;
    v = (v | (v << 4)) & 0x030C30C3u;
    v = (v | (v << 2)) & 0x09249249u;
  } else if (dims == 2) {  // 16 bits -> every second bit of 32
    v &= 0xFFFFu;
    v = (v | (v << 8)) & 0x00FF00FFu;
    v = (v | (v << 4)) & 0x0F0F0F0Fu;
    v = (v | (v << 2)) & 0x33333333u;
    v = (v | (v << 1)) & 0x55555555u;
  }
  return v;
}

struct MortonFrame {
  float lo[kSortDims];
  float scale[kSortDims];  // (2^bits - 1) / extent, 0 for a flat coordinate
  int dims;
  int bits;
};

// Key (Morton code << 32 | index) of every point; entries count .. n_pow2 get the largest key.
__global__ void __launch_bounds__(256) morton_keys_kernel(const float* pts, int64_t count,
                                                          int32_t d, const MortonFrame F,
                                                          uint64_t* keys, int64_t n_pow2) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= n_pow2) return;
  if (j >= count) {
    keys[j] = ~0ull;
    return;
  }
  uint32_t code = 0;
  const uint32_t qmax = (1u << F.bits) - 1u;
  for (int k = 0; k < F.dims; ++k) {
    float q = (pts[j * d + k] - F.lo[k]) * F.scale[k];
    q = fminf(fmaxf(q, 0.0f), static_cast<float>(qmax));
    code |= spread_bits(static_cast<uint32_t>(q), F.dims) << k;
  }
  keys[j] = (static_cast<uint64_t>(code) << 32) | static_cast<uint64_t>(j);
}

__device__ __forceinline__ void cmp_swap(uint64_t& a, uint64_t& b, bool ascending) {
  if ((a > b) == ascending) {
    const uint64_t t = a;
    a = b;
    b = t;
  }
}

// Bitonic stages with sizes k <= kSortSmem (first call: all of them; later calls: the
// strides j < kSortSmem of merge size k), in shared memory, one block per kSortSmem keys.
__global__ void __launch_bounds__(kSortBlock) bitonic_smem_kernel(uint64_t* keys, int64_t k_merge) {
  __shared__ uint64_t s[kSortSmem];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kSortSmem;
  const int t = threadIdx.x;
  s[t] = keys[base + t];
  s[t + kSortBlock] = keys[base + t + kSortBlock];
  __syncthreads();
  const int64_t k_lo = k_merge > 0 ? k_merge : 2;
  const int64_t k_hi = k_merge > 0 ? k_merge : kSortSmem;
  for (int64_t k = k_lo; k <= k_hi; k <<= 1) {
    for (int64_t j = (k_merge > 0 ? kSortSmem / 2 : k / 2); j > 0; j >>= 1) {
      // thread t handles the pair (i, i + j) with i = 2t - (t mod j)
      const int i = 2 * t - (t & static_cast<int>(j - 1));
      const bool asc = ((base + i) & k) == 0;
      cmp_swap(s[i], s[i + j], asc);
      __syncthreads();
    }
  }
  keys[base + t] = s[t];
  keys[base + t + kSortBlock] = s[t + kSortBlock];
}

// One bitonic step with stride j >= kSortSmem over all n_pow2 keys.
__global__ void __launch_bounds__(256) bitonic_global_kernel(uint64_t* keys, int64_t n_pow2,
                                                             int64_t k, int64_t j) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n_pow2 / 2) return;
  const int64_t i = 2 * t - (t & (j - 1));
  const bool asc = (i & k) == 0;
  uint64_t a = keys[i], b = keys[i + j];
  if ((a > b) == asc) {
    keys[i] = b;
    keys[i + j] = a;
  }
}

// The permutation (original index of each sorted position) and the sorted Morton codes.
__global__ void __launch_bounds__(256) perm_from_keys_kernel(const uint64_t* keys, int64_t count,
                                                             int* perm, unsigned* codes) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= count) return;
  const uint64_t k = keys[j];
  perm[j] = static_cast<int>(k & 0xFFFFFFFFull);
  codes[j] = static_cast<unsigned>(k >> 32);
}

// Group records of the screened passes (D <= 3): per 256-point tile, 16 groups of 16
// consecutive points (8 key pairs, the pass's unit of work), each kGroupRecFloats floats
// [lo_0 lo_1 lo_2 hi_0 hi_1 hi_2 Hmax pad], a tile's records contiguous (one bulk copy).
constexpr int kGroupKeys = 16;
constexpr int kGroupRecFloats = 8;
constexpr int kTileGroupFloats = (256 / kGroupKeys) * kGroupRecFloats;  // 128 floats, 512 B

// Bounding box (all D coordinates) of each 256-point tile of a packed cloud, stored by
// component: box[k * T + t] = lo_k, box[(D + k) * T + t] = hi_k of tile t (T tiles), so that
// a warp scanning consecutive tiles reads each component in one coalesced request. Only
// real points count. With gsum (D <= 3) the boxes of the tile's 16-point groups go to their
// group records as well.
template <int D>
__global__ void __launch_bounds__(256) tile_box_kernel(const float* keys, int64_t count, float* box,
                                                       int64_t T, float* gsum) {
  constexpr int KP = ((2 * (D + 1) + 3) / 4) * 4;
  const int64_t t = blockIdx.x;
  const int64_t j = t * 256 + threadIdx.x;
  __shared__ float red[2][D][8];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < D; ++k) {
    float v = INFINITY, u = -INFINITY;
    if (j < count) {
      v = u = keys[(j >> 1) * KP + 2 * k + (j & 1)];
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
      u = fmaxf(u, __shfl_xor_sync(0xffffffffu, u, o));
    }
    if (D <= 3 && gsum && (lane & 15) == 0) {
      float* rec = gsum + (t * (256 / kGroupKeys) + threadIdx.x / kGroupKeys) * kGroupRecFloats;
      rec[k] = v;
      rec[3 + k] = u;
    }
    v = fminf(v, __shfl_xor_sync(0xffffffffu, v, 16));
    u = fmaxf(u, __shfl_xor_sync(0xffffffffu, u, 16));
    if (lane == 0) {
      red[0][k][w] = v;
      red[1][k][w] = u;
    }
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int k = threadIdx.x;
    float v = INFINITY, u = -INFINITY;
    for (int q = 0; q < 8; ++q) {
      v = fminf(v, red[0][k][q]);
      u = fmaxf(u, red[1][k][q]);
    }
    box[k * T + t] = v;
    box[(D + k) * T + t] = u;
  }
}

// Largest key bias H of each 256-point tile of a packed cloud (kLogZero if none is real);
// with gsum (D <= 3) also of each 16-point group, into its group record.
template <int D>
__global__ void __launch_bounds__(256) tile_hmax_kernel(const float* keys, int64_t count,
                                                        float* hmax, float* gsum) {
  constexpr int KP = ((2 * (D + 1) + 3) / 4) * 4;
  const int64_t T = blockIdx.x;
  const int64_t j = T * 256 + threadIdx.x;
  __shared__ float red[8];
  float h = kLogZero;
  if (j < count) h = keys[(j >> 1) * KP + 2 * D + (j & 1)];
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) h = fmaxf(h, __shfl_xor_sync(0xffffffffu, h, o));
  if (D <= 3 && gsum && (threadIdx.x & 15) == 0)
    gsum[(T * (256 / kGroupKeys) + threadIdx.x / kGroupKeys) * kGroupRecFloats + 6] = h;
  h = fmaxf(h, __shfl_xor_sync(0xffffffffu, h, 16));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = h;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int q = 1; q < 8; ++q) m = fmaxf(m, red[q]);
    hmax[T] = m;
  }
}

// Super-tiles: runs of kSuper consecutive tiles (2048 points), summarised the same way, so
// that screening can reject a whole run with one test. One thread per super-tile; `nc`
// components of stride T (tiles) and S (super-tiles); `take_max` picks max over the run
// (biases, upper box corners) or min (lower corners) per component.
constexpr int kSuper = 8;

__global__ void __launch_bounds__(256) super_reduce_kernel(const float* v, int64_t T, float* out,
                                                           int64_t S, int nc, int n_min) {
  const int64_t s = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (s >= S) return;
  const int64_t t0 = s * kSuper, t1 = t0 + kSuper < T ? t0 + kSuper : T;
  for (int c = 0; c < nc; ++c) {
    const bool take_min = c < n_min;
    float r = take_min ? INFINITY : -INFINITY;
    for (int64_t t = t0; t < t1; ++t) {
      const float x = v[c * T + t];
      r = take_min ? fminf(r, x) : fmaxf(r, x);
    }
    out[c * S + s] = r;
  }
}

}  // namespace fs
