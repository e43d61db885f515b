// fs_transport.cuh -- elementwise kernels of the Hessian-vector product (FlashSinkhorn
// summary, section 3: an HVP decomposed into transport-vector and transport-matrix
// products). The products themselves are streaming passes (lse_pass_kernel in kModePay and
// kModeDiff); these kernels form their inputs and combine their outputs.
//
// At the plan P of (F(g), g) (rows sum to a) and for one vector v_i per point x_i:
//   r_i = sum_j P_ij 2 (x_i - y_j).v_i = v_i . grad_i,   grad_i = 2 (a_i x_i - sum_j P_ij y_j)
//   s_j = sum_i P_ij 2 (x_i - y_j).v_i = 2 [sum_i P_ij (x_i - c).v_i - (y_j - c).sum_i P_ij v_i]
//   [diag(P 1)  P ; P^T  diag(P^T 1)] (df, dg) = (r, s)          (conjugate gradients)
//   (H v)_i = 2 a_i v_i + (2/eps) [df_i grad_i / 2 - sum_j P_ij (dg_j + 2 (y_j - x_i).v_i)(y_j - x_i)]
// with c the centre of the clouds' box (it cancels; it only keeps the column sums small).
#pragma once

#include "fs_kernels.cuh"

namespace fs {

// r_i = v_i . grad_i and the payload of the column pass, (1, (x_i - c).v_i, v_i).
__global__ void __launch_bounds__(256) hvp_row_prep_kernel(const float* x, const float* v,
                                                           const float* grad, int64_t n,
                                                           int32_t d, float c0, float c1,
                                                           float c2, float* r, float* colpay) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float rv = 0.0f, xv = 0.0f;
  float* cp = colpay + i * (d + 2);
  for (int k = 0; k < d; ++k) {
    const float vk = v[i * d + k];
    const float ck = k == 0 ? c0 : (k == 1 ? c1 : (k == 2 ? c2 : 0.0f));
    rv = fmaf(vk, grad[i * d + k], rv);
    xv = fmaf(x[i * d + k] - ck, vk, xv);
    cp[2 + k] = vk;
  }
  cp[0] = 1.0f;
  cp[1] = xv;
  r[i] = rv;
}

// s_j = 2 [coldata_j1 - (y_j - c).coldata_j(2..)] and the column sums coldata_j0.
__global__ void __launch_bounds__(256) hvp_col_rhs_kernel(const float* y, const float* coldata,
                                                          int64_t m, int32_t d, float c0,
                                                          float c1, float c2, float* s,
                                                          float* csum) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= m) return;
  const float* cd = coldata + j * (d + 2);
  float t = cd[1];
  for (int k = 0; k < d; ++k) {
    const float ck = k == 0 ? c0 : (k == 1 ? c1 : (k == 2 ? c2 : 0.0f));
    t = fmaf(-(y[j * d + k] - ck), cd[2 + k], t);
  }
  s[j] = 2.0f * t;
  csum[j] = cd[0];
}

// Block sum of v.w (or v.v) into a float64 accumulator.
__global__ void __launch_bounds__(256) cg_dot_kernel(const float* v, const float* w, int64_t len,
                                                     double* out) {
  __shared__ double sh[8];
  double acc = 0.0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < len;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    acc += static_cast<double>(v[i]) * static_cast<double>(w[i]);
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    acc = threadIdx.x < (blockDim.x >> 5) ? sh[threadIdx.x] : 0.0;
    acc = warp_sum(acc);
    if (threadIdx.x == 0) atomicAdd(out, acc);
  }
}

// Block sums of a vector's two parts (rows [0, n) and columns [n, n + m)).
__global__ void __launch_bounds__(256) cg_split_sum_kernel(const float* v, int64_t n, int64_t m,
                                                           double* out) {
  __shared__ double sh[2][8];
  double a = 0.0, b = 0.0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n + m;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (i < n)
      a += v[i];
    else
      b += v[i];
  }
  a = warp_sum(a);
  b = warp_sum(b);
  if ((threadIdx.x & 31) == 0) {
    sh[0][threadIdx.x >> 5] = a;
    sh[1][threadIdx.x >> 5] = b;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const bool in = threadIdx.x < (blockDim.x >> 5);
    a = warp_sum(in ? sh[0][threadIdx.x] : 0.0);
    b = warp_sum(in ? sh[1][threadIdx.x] : 0.0);
    if (threadIdx.x == 0) {
      atomicAdd(&out[0], a);
      atomicAdd(&out[1], b);
    }
  }
}

// Removes the gauge direction (1, -1) from (r, s): r -= delta, s += delta with
// delta = (sum r - sum s) / (n + m), read from the two sums.
__global__ void __launch_bounds__(256) cg_project_kernel(float* v, int64_t n, int64_t m,
                                                         const double* sums) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n + m) return;
  const float delta = static_cast<float>((sums[0] - sums[1]) / static_cast<double>(n + m));
  v[i] += i < n ? -delta : delta;
}

// Ap = (a o u + P w, csum o w + P^T u) from the two transport products.
__global__ void __launch_bounds__(256) cg_apply_kernel(const float* p, const float* a, float a_uni,
                                                       const float* csum, const float* pw,
                                                       const float* ptu, int64_t n, int64_t m,
                                                       float* ap) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) {
    ap[i] = fmaf(a ? a[i] : a_uni, p[i], pw[i]);
  } else if (i < n + m) {
    const int64_t j = i - n;
    ap[i] = fmaf(csum[j], p[i], ptu[j]);
  }
}

// z += alpha p, r -= alpha Ap.
__global__ void __launch_bounds__(256) cg_step_kernel(float* z, float* r, const float* p,
                                                      const float* ap, int64_t len, float alpha) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= len) return;
  z[i] = fmaf(alpha, p[i], z[i]);
  r[i] = fmaf(-alpha, ap[i], r[i]);
}

// p = r + beta p.
__global__ void __launch_bounds__(256) cg_dir_kernel(float* p, const float* r, int64_t len,
                                                     float beta) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= len) return;
  p[i] = fmaf(beta, p[i], r[i]);
}

// 2 v (the row vectors of the difference pass).
__global__ void __launch_bounds__(256) scale_kernel(const float* v, int64_t len, float s,
                                                    float* out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < len) out[i] = s * v[i];
}

// (H v)_i = 2 a_i v_i + (2/eps) [df_i grad_i / 2 - diffsum_i].
__global__ void __launch_bounds__(256) hvp_final_kernel(const float* v, const float* a, float a_uni,
                                                        const float* df, const float* grad,
                                                        const float* diffsum, int64_t n,
                                                        int32_t d, double two_over_eps,
                                                        float* out) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n * d) return;
  const int64_t i = t / d;
  const double ai = a ? static_cast<double>(a[i]) : static_cast<double>(a_uni);
  const double inner = 0.5 * static_cast<double>(df[i]) * grad[t] - static_cast<double>(diffsum[t]);
  out[t] = static_cast<float>(2.0 * ai * v[t] + two_over_eps * inner);
}

}  // namespace fs
