// The light HBM-bound passes around the GEMMs: gain fold, SwiGLU backward
// with its row statistic, and the column reduce of the dg partials.  All use
// 16-byte vector accesses.  (The row reduce of the partial sums of squares,
// the "very light auxiliary reduction" of the kucoin.com (ru) CODA article,
// section «В «Финале» спрятаны сокровища», runs in the gate/up GEMM's
// epilogue, see swiglu_row_scale in coda_gemm.cuh.)
#pragma once

#include "coda_ptx.cuh"

namespace coda {

// W2g[n, j] = bf16(g[j] * W2[n, j]); 8 elements per thread, d % 8 == 0.
// The RMSNorm gain as diag(g) folded into the second GEMM's weight (the
// toolin.ai five-primitive table lists the RMSNorm weight broadcast as a
// vector-load primitive; folding it once per weight update removes it from
// the epilogue entirely).
constexpr int FOLD_UNROLL = 4;  // independent 16-byte loads in flight per thread
__global__ void fold_gain_kernel(const __nv_bfloat16* __restrict__ W2, const __nv_bfloat16* __restrict__ g,
                                 __nv_bfloat16* __restrict__ W2g, int d, long long n_vec8) {
  griddep_wait();
  const int dv = d / 8;  // 8-element vectors per row
  const long long S = (long long)gridDim.x * blockDim.x;
  const int s_mod = (int)(S % dv);
  long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  int jv = (int)(v % dv);  // column vector of v; advanced by S mod dv per step
  for (; v < n_vec8; v += FOLD_UNROLL * S) {
    // The step's loads of W2 and of g are independent of its stores, so all
    // are issued first.  g (d values, reused by every row) goes through L1.
    uint4 w[FOLD_UNROLL], gq[FOLD_UNROLL];
#pragma unroll
    for (int u = 0; u < FOLD_UNROLL; ++u) {
      const long long vu = v + u * S;
      if (vu < n_vec8) {
        w[u] = ldg_nc_v4(W2 + vu * 8);
        gq[u] = ldg_nc_v4_l1(g + jv * 8);
      }
      jv += s_mod;
      if (jv >= dv) jv -= dv;
    }
#pragma unroll
    for (int u = 0; u < FOLD_UNROLL; ++u) {
      const long long vu = v + u * S;
      if (vu >= n_vec8) break;
      float f[8], gg[8];
      unpack8(w[u], f);
      unpack8(gq[u], gg);
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] *= gg[i];
      stg_v4(W2g + vu * 8, pack8(f));
    }
  }
}

// c_i = (r_i^2 / d) sum_t Pc[i, t]: the RMSNorm backward's row coefficient
// from the per-tile partials of the down-projection dgrad's epilogue.
__global__ void rowcoef_reduce_kernel(const float* __restrict__ Pc, int T, const float* __restrict__ r,
                                      float* __restrict__ c, int M, float inv_d) {
  griddep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M) return;
  const float* row = Pc + (size_t)i * T;
  float s = 0.f;
  for (int t = 0; t < T; ++t) s += row[t];
  c[i] = r[i] * r[i] * inv_d * s;
}

template <int THREADS>
__device__ __forceinline__ float block_sum(float v, float* scratch) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x / 32;
  if ((threadIdx.x & 31) == 0) scratch[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < 32) {
    t = threadIdx.x < THREADS / 32 ? scratch[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  }
  return t;  // valid in thread 0
}

// SwiGLU backward fused with the RMSNorm backward's row statistic, one block
// per token row (F % 8 == 0):
//   sigma = sigmoid(a); da = dY b sigma (1 + a (1 - sigma)); db = dY a sigma
//   dA'  = bf16(r_i [da | db])            (the dn and dW2 GEMMs' left operand)
//   c_i  = (r_i^2 / d) * sum_c (da a + db b)
// c_i is the coefficient of the -c_i H_ij term of dH: with A = [a | b] the
// pre-activations, sum_c dA_ic A_ic equals r_i sum_k dn_ik H_ik, so the whole
// RMSNorm correction is a block-local epilogue term of the dn GEMM.
constexpr int ROWSTAT_THREADS = 256;
__global__ void __launch_bounds__(ROWSTAT_THREADS)
    swiglu_bwd_rowstat_kernel(const __nv_bfloat16* __restrict__ dY, const __nv_bfloat16* __restrict__ AB,
                              const float* __restrict__ r, __nv_bfloat16* __restrict__ dAp,
                              float* __restrict__ c, int F, float inv_d) {
  __shared__ float scratch[32];
  griddep_wait();
  const int row = blockIdx.x;
  const __nv_bfloat16* dy = dY + (size_t)row * F;
  const __nv_bfloat16* a = AB + (size_t)row * 2 * F;
  const __nv_bfloat16* b = a + F;
  __nv_bfloat16* oa = dAp + (size_t)row * 2 * F;
  __nv_bfloat16* ob = oa + F;
  const float rr = r[row];
  float acc = 0.f;
  for (int v = threadIdx.x; v < F / 8; v += ROWSTAT_THREADS) {
    float fy[8], fa[8], fb[8], da[8], db[8];
    unpack8(ldg_nc_v4(dy + 8 * v), fy);
    unpack8(ldg_nc_v4(a + 8 * v), fa);
    unpack8(ldg_nc_v4(b + 8 * v), fb);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float s = sigmoid_f(fa[i]);
      da[i] = fy[i] * fb[i] * s * (1.f + fa[i] * (1.f - s));
      db[i] = fy[i] * fa[i] * s;
      acc = fmaf(da[i], fa[i], acc);
      acc = fmaf(db[i], fb[i], acc);
      da[i] *= rr;
      db[i] *= rr;
    }
    stg_v4(oa + 8 * v, pack8(da));
    stg_v4(ob + 8 * v, pack8(db));
  }
  const float tot = block_sum<ROWSTAT_THREADS>(acc, scratch);
  if (threadIdx.x == 0) c[row] = rr * rr * inv_d * tot;
}

// dg_j = sum_t Pg[t, j]: reduce the dn GEMM's per-32-row column partials.
// One block per 32 columns; warp w sums rows w, w+8, ... (lane = column, so
// each warp load is one 128-byte line), then the 8 warp sums are added in a
// fixed order, so the result is bit-reproducible.
constexpr int COLRED_THREADS = 256;
__global__ void __launch_bounds__(COLRED_THREADS)
    col_reduce_kernel(const float* __restrict__ Pg, int rows, int d, float* __restrict__ dg) {
  __shared__ float part[COLRED_THREADS / 32][32];
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const int j = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (j < d) {
#pragma unroll 4
    for (int t = w; t < rows; t += COLRED_THREADS / 32) s += Pg[(size_t)t * d + j];
  }
  part[w][lane] = s;
  __syncthreads();
  if (w == 0 && j < d) {
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < COLRED_THREADS / 32; ++k) tot += part[k][lane];
    dg[j] = tot;
  }
}

// Inverse RoPE of the q/k gradient (rotation by -pos * base^(-2j/hd)) and a
// copy of the v gradient: dpre = R(pos)^T dQKV, the A operand of the backward
// GEMMs.  A rotation item is one row, one slice of 8 pairs (j0 .. j0 + 7) and
// up to ROPE_HEADS rotated heads; the heads share the slice's angles, so its
// 8 sines and cosines are computed once for all of them, and the heads' loads
// are issued in groups of 4 before any store.  A copy item is 32 v columns,
// four 16-byte loads issued before their stores.
constexpr int ROPE_HEADS = 8;
constexpr int ROPE_COPY_COLS = 32;
__global__ void rope_unrotate_kernel(const __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dpre,
                                     int M, int ncols, int head_dim, int rot_cols, int seq_len, float rope_k) {
  griddep_wait();
  const int half = head_dim / 2;
  const int slices = half / 8;
  const int rot_heads = rot_cols / head_dim;
  const int groups = (rot_heads + ROPE_HEADS - 1) / ROPE_HEADS;
  const long long rot_total = (long long)M * slices * groups;
  const int copy_per_row = (ncols - rot_cols) / ROPE_COPY_COLS;  // v heads are multiples of 64 columns
  const long long total = rot_total + (long long)M * copy_per_row;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long it = (long long)blockIdx.x * blockDim.x + threadIdx.x; it < total; it += stride) {
    if (it >= rot_total) {
      const long long ci = it - rot_total;
      const int row = (int)(ci / copy_per_row);
      const size_t off =
          (size_t)row * ncols + rot_cols + (size_t)(ci - (long long)row * copy_per_row) * ROPE_COPY_COLS;
      uint4 v[ROPE_COPY_COLS / 8];
#pragma unroll
      for (int k = 0; k < ROPE_COPY_COLS / 8; ++k) v[k] = ldg_nc_v4(dq + off + 8 * k);
#pragma unroll
      for (int k = 0; k < ROPE_COPY_COLS / 8; ++k) stg_v4(dpre + off + 8 * k, v[k]);
      continue;
    }
    // it = (row * groups + group) * slices + slice: neighbouring threads take
    // neighbouring slices of one head group, so their 16-byte accesses abut.
    const int sl = (int)(it % slices);
    const long long rg = it / slices;
    const int grp = (int)(rg % groups);
    const int row = (int)(rg / groups);
    const int j0 = sl * 8;
    const float pos = (float)(row % seq_len);
    float sn[8], cs[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sincosf(pos * exp2f((float)(j0 + i) * rope_k), &sn[i], &cs[i]);
    const size_t base = (size_t)row * ncols + j0;
    const int h_end = min(rot_heads, (grp + 1) * ROPE_HEADS);
#pragma unroll 1
    for (int h0 = grp * ROPE_HEADS; h0 < h_end; h0 += 4) {
      uint4 q1[4], q2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (h0 + k < h_end) {
          const size_t c1 = base + (size_t)(h0 + k) * head_dim;
          q1[k] = ldg_nc_v4(dq + c1);
          q2[k] = ldg_nc_v4(dq + c1 + half);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (h0 + k >= h_end) break;
        float x1[8], x2[8];
        unpack8(q1[k], x1);
        unpack8(q2[k], x2);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float y1 = x1[i] * cs[i] + x2[i] * sn[i];
          const float y2 = x2[i] * cs[i] - x1[i] * sn[i];
          x1[i] = y1;
          x2[i] = y2;
        }
        const size_t c1 = base + (size_t)(h0 + k) * head_dim;
        stg_v4(dpre + c1, pack8(x1));
        stg_v4(dpre + c1 + half, pack8(x2));
      }
    }
  }
}

// Cross-entropy row reduce, one warp per row: merge the tiles' (max, sum exp)
// partials, lse = max + log(sum), loss = lse - target logit (the target logit
// is NaN when the target was out of range, so the loss is too).
__device__ __forceinline__ void lse_merge(float& m, float& s, float om, float os) {
  if (om == -INFINITY) return;
  if (m == -INFINITY) {
    m = om;
    s = os;
    return;
  }
  const float nm = fmaxf(m, om);
  s = s * expf(m - nm) + os * expf(om - nm);
  m = nm;
}

__global__ void xent_reduce_kernel(const float2* __restrict__ part, int T, const float* __restrict__ tlogit,
                                   float* __restrict__ lse, float* __restrict__ loss, int M) {
  griddep_wait();
  const int row = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  float m = -INFINITY, s = 0.f;
  for (int t = lane; t < T; t += 32) {
    const float2 q = part[(size_t)row * T + t];
    lse_merge(m, s, q.x, q.y);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, o);
    const float os = __shfl_xor_sync(0xffffffffu, s, o);
    lse_merge(m, s, om, os);
  }
  if (lane == 0) {
    const float l = m + logf(s);
    lse[row] = l;
    loss[row] = l - tlogit[row];
  }
}

// Self-test of the device-side failure path: one warp waits, with the same
// bounded wait the GEMM pipeline uses, on an mbarrier that nothing arrives on.
// The wait gives up after limit_ns, records CODA_ERR_DEVICE_TIMEOUT and the
// detail word in the status word, and the kernel returns normally.
constexpr uint32_t kSelftestKernelId = 0x3F;
__global__ void selftest_wait_timeout_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtl ctl{&abort_flag, status, limit_ns, kSelftestKernelId};
  if (threadIdx.x == 0) mbar_wait(&bar, 0, ctl, 0, kWaitFull);
  __syncthreads();
}

}  // namespace coda
