// The unfused comparison sequence: the same block computed the way an
// operator-by-operator framework runs it, one kernel per operation with every
// intermediate written to and read back from HBM (the "operator boundaries"
// the pages blame for the memory traffic: toolin.ai CODA article, section 課題;
// kucoin.com (ru), section «Налог на лень»).  Used for measurement and for the
// error comparison only; the GEMMs are the same tcgen05 kernels with the plain
// store epilogue, so the difference measured is the fusion alone.
#pragma once

#include "coda_aux.cuh"

namespace coda {

constexpr int UNF_THREADS = 256;

// H = bf16(T + R), 8 elements per thread (n % 8 == 0).
__global__ void unf_residual_add_kernel(const __nv_bfloat16* __restrict__ T, const __nv_bfloat16* __restrict__ R,
                                        __nv_bfloat16* __restrict__ H, long long n_vec8) {
  griddep_wait();
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < n_vec8; v += stride) {
    float t[8], r[8];
    unpack8(ldg_nc_v4(T + 8 * v), t);
    unpack8(ldg_nc_v4(R + 8 * v), r);
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] += r[i];
    stg_v4(H + 8 * v, pack8(t));
  }
}

// RMSNorm with gain, one block per row: r_i = 1/sqrt(mean_j H_ij^2 + eps),
// U = bf16(H_ij r_i g_j).  d % 8 == 0.
__global__ void __launch_bounds__(UNF_THREADS)
    unf_rmsnorm_fwd_kernel(const __nv_bfloat16* __restrict__ H, const __nv_bfloat16* __restrict__ g,
                           __nv_bfloat16* __restrict__ U, float* __restrict__ r, int d, float eps) {
  __shared__ float scratch[32];
  __shared__ float r_sh;
  griddep_wait();
  const int row = blockIdx.x;
  const __nv_bfloat16* h = H + (size_t)row * d;
  float ss = 0.f;
  for (int v = threadIdx.x; v < d / 8; v += UNF_THREADS) {
    float f[8];
    unpack8(ldg_nc_v4(h + 8 * v), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
  const float tot = block_sum<UNF_THREADS>(ss, scratch);
  if (threadIdx.x == 0) {
    r_sh = rsqrtf(tot / (float)d + eps);
    r[row] = r_sh;
  }
  __syncthreads();
  const float rr = r_sh;
  for (int v = threadIdx.x; v < d / 8; v += UNF_THREADS) {
    float f[8], gg[8];
    unpack8(ldg_nc_v4(h + 8 * v), f);
    unpack8(ldg_nc_v4(g + 8 * v), gg);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = f[i] * rr * gg[i];
    stg_v4(U + (size_t)row * d + 8 * v, pack8(f));
  }
}

// Y = bf16(silu(a) * b) from A = [a | b] (bf16 [M, 2F]).  F % 8 == 0.
__global__ void unf_swiglu_fwd_kernel(const __nv_bfloat16* __restrict__ A, __nv_bfloat16* __restrict__ Y, int F,
                                      long long n_vec8 /* M * F / 8 */) {
  griddep_wait();
  const long long stride = (long long)gridDim.x * blockDim.x;
  const int fv = F / 8;
  for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < n_vec8; v += stride) {
    const long long row = v / fv;
    const int c = (int)(v - row * fv) * 8;
    float a[8], b[8];
    unpack8(ldg_nc_v4(A + row * 2 * F + c), a);
    unpack8(ldg_nc_v4(A + row * 2 * F + F + c), b);
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = a[i] * sigmoid_f(a[i]) * b[i];
    stg_v4(Y + row * F + c, pack8(a));
  }
}

// dA = [da | db] (bf16) from dY and A = [a | b].
__global__ void unf_swiglu_bwd_kernel(const __nv_bfloat16* __restrict__ dY, const __nv_bfloat16* __restrict__ A,
                                      __nv_bfloat16* __restrict__ dA, int F, long long n_vec8) {
  griddep_wait();
  const long long stride = (long long)gridDim.x * blockDim.x;
  const int fv = F / 8;
  for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < n_vec8; v += stride) {
    const long long row = v / fv;
    const int c = (int)(v - row * fv) * 8;
    float dy[8], a[8], b[8];
    unpack8(ldg_nc_v4(dY + row * F + c), dy);
    unpack8(ldg_nc_v4(A + row * 2 * F + c), a);
    unpack8(ldg_nc_v4(A + row * 2 * F + F + c), b);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float s = sigmoid_f(a[i]);
      const float da = dy[i] * b[i] * s * (1.f + a[i] * (1.f - s));
      const float db = dy[i] * a[i] * s;
      a[i] = da;
      b[i] = db;
    }
    stg_v4(dA + row * 2 * F + c, pack8(a));
    stg_v4(dA + row * 2 * F + F + c, pack8(b));
  }
}

// RMSNorm backward, one block per row, from du = dA W2 (bf16):
//   dn = du * g;  s_i = sum_k dn_ik H_ik;  dH = r dn - (r^3/d) s_i H (+ dH_in).
__global__ void __launch_bounds__(UNF_THREADS)
    unf_rmsnorm_bwd_kernel(const __nv_bfloat16* __restrict__ du, const __nv_bfloat16* __restrict__ H,
                           const __nv_bfloat16* __restrict__ g, const float* __restrict__ r,
                           const __nv_bfloat16* __restrict__ dH_in, __nv_bfloat16* __restrict__ dH, int d) {
  __shared__ float scratch[32];
  __shared__ float s_sh;
  griddep_wait();
  const int row = blockIdx.x;
  const size_t off = (size_t)row * d;
  float acc = 0.f;
  for (int v = threadIdx.x; v < d / 8; v += UNF_THREADS) {
    float u[8], h[8], gg[8];
    unpack8(ldg_nc_v4(du + off + 8 * v), u);
    unpack8(ldg_nc_v4(H + off + 8 * v), h);
    unpack8(ldg_nc_v4(g + 8 * v), gg);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc = fmaf(u[i] * gg[i], h[i], acc);
  }
  const float tot = block_sum<UNF_THREADS>(acc, scratch);
  if (threadIdx.x == 0) s_sh = tot;
  __syncthreads();
  const float rr = r[row];
  const float coef = rr * rr * rr / (float)d * s_sh;
  for (int v = threadIdx.x; v < d / 8; v += UNF_THREADS) {
    float u[8], h[8], gg[8], e[8];
    unpack8(ldg_nc_v4(du + off + 8 * v), u);
    unpack8(ldg_nc_v4(H + off + 8 * v), h);
    unpack8(ldg_nc_v4(g + 8 * v), gg);
    if (dH_in != nullptr) unpack8(ldg_nc_v4(dH_in + off + 8 * v), e);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      u[i] = rr * u[i] * gg[i] - coef * h[i];
      if (dH_in != nullptr) u[i] += e[i];
    }
    stg_v4(dH + off + 8 * v, pack8(u));
  }
}

// dg_j = sum_i du_ij H_ij r_i: column partial sums over blocks of 64 rows,
// then the column reduce.  One thread per column, d % 8 == 0 not required.
constexpr int UNF_DG_ROWS = 64;
__global__ void unf_dg_partial_kernel(const __nv_bfloat16* __restrict__ du, const __nv_bfloat16* __restrict__ H,
                                      const float* __restrict__ r, float* __restrict__ part, int M, int d) {
  griddep_wait();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  const int r0 = blockIdx.y * UNF_DG_ROWS;
  const int r1 = min(M, r0 + UNF_DG_ROWS);
  float s = 0.f;
  for (int i = r0; i < r1; ++i)
    s = fmaf(__bfloat162float(du[(size_t)i * d + j]) * r[i], __bfloat162float(H[(size_t)i * d + j]), s);
  part[(size_t)blockIdx.y * d + j] = s;
}

}  // namespace coda
