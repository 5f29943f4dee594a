// gptq.cuh -- GPTQ (Algorithm 1 of "GPTQ: Accurate Post-Training Quantization
// for Generative Pre-trained Transformers", sections 2-3) on the GPU, the
// baseline the ADMM-Q objective is reported against.
//
// Layout: W_hat and codes are [d_out][d_in] (one output row per weight row),
// so the algorithm's columns are our input columns j = 0 .. d_in - 1.  With
// R the upper Cholesky factor of H^-1 (R^T R = H^-1, H = X^T X + lambda I),
// columns are visited in blocks of B:
//   for j in block:  q_j = clamp(rint(w_j / s) + z, 0, L)   (grid of w's group)
//                    e_j = (w_j - s (q_j - z)) / R_jj
//                    w_{j..b-1} -= e_j R_{j, j..b-1}
//   then             W[:, b:] -= E R[block, b:]      (a plain fp64 GEMM)
// The grid (scale, zero per row and group) is fixed: the min/max grid of
// W_hat, the same one RTN uses.  Everything runs in float64 with explicitly
// rounded operations, in the order the algorithm states.
//
// Included by admmq.cu inside its internal namespace, after the weight-load
// helper load_w<T>.
#pragma once
#include <stdint.h>

// Per (row, group): the min/max grid of W_hat (float32, the RTN rule) and the
// float64 working copy of the row segment.
template <typename T>
__global__ void k_gptq_start(const T* __restrict__ W, int m, int d, int g, int L,
                             float* __restrict__ scale, float* __restrict__ zero,
                             double* __restrict__ Wd) {
  const int ngr = d / g;
  const long long total = (long long)m * ngr;
  const float Lf = (float)L;
  for (long long gi = blockIdx.x * (long long)blockDim.x + threadIdx.x; gi < total;
       gi += (long long)gridDim.x * blockDim.x) {
    const long long row = gi / ngr;
    const long long base = row * d + (gi - row * ngr) * g;
    float mn = 0.f, mx = 0.f;
    for (int e = 0; e < g; ++e) {
      const float y = load_w<T>(W, base + e);
      mn = fminf(mn, y);
      mx = fmaxf(mx, y);
      Wd[base + e] = (double)y;
    }
    float s = __fdiv_rn(__fsub_rn(mx, mn), Lf), z;
    if (s == 0.f) {
      s = 1.f;
      z = 0.f;
    } else {
      z = __fadd_rn(rintf(__fdiv_rn(-mn, s)), 0.f);
    }
    scale[gi] = s;
    zero[gi] = z;
  }
}

// H (+ lambda I) in float64 from the fp32 Gram and the damping term.
__global__ void k_gptq_hessian(const float* __restrict__ G, int d, const double* __restrict__ lam,
                               double* __restrict__ Hd) {
  const long long total = (long long)d * d;
  const double l = *lam;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long i = idx / d;
    Hd[idx] = (double)G[idx] + (idx - i * d == i ? l : 0.0);
  }
}

// One block of columns [a, a + bw), bw <= 128 and a multiple of 32: a warp per
// output row, lane l holding columns a + l + 32k.  The column loop is
// sequential; e_j goes from the lane that owns column j to the others by a
// shuffle.  R is row-major upper (R[j][c], c >= j).  Writes the codes of the
// block and E[row][j - a].
__global__ void __launch_bounds__(256) k_gptq_block(double* __restrict__ Wd, const double* __restrict__ R,
                                                    const float* __restrict__ scale,
                                                    const float* __restrict__ zero, int m, int d, int g,
                                                    int L, int a, int bw, uint8_t* __restrict__ codes,
                                                    double* __restrict__ E, int ldE) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= m) return;  // whole warps only: m rows, blockDim a multiple of 32
  const int ngr = d / g;
  const double Ld = (double)L;
  double w[4];
  uint32_t q[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int cc = lane + 32 * k;
    w[k] = cc < bw ? Wd[row * d + a + cc] : 0.0;
    q[k] = 0u;
  }
  for (int jj = 0; jj < bw; ++jj) {
    const int kj = jj >> 5, owner = jj & 31;
    const long long j = a + jj;
    double e = 0.0;
    if (lane == owner) {
      double wj = w[0];
#pragma unroll
      for (int k = 1; k < 4; ++k)
        if (k == kj) wj = w[k];
      const long long gi = row * ngr + j / g;
      const double s = (double)scale[gi], z = (double)zero[gi];
      double c = __dadd_rn(rint(__ddiv_rn(wj, s)), z);
      c = fmin(fmax(c, 0.0), Ld);
      const double qd = __dmul_rn(s, __dsub_rn(c, z));
      e = __ddiv_rn(__dsub_rn(wj, qd), R[j * d + j]);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (k == kj) q[k] = (uint32_t)c;
      E[row * ldE + jj] = e;
    }
    e = __shfl_sync(0xffffffffu, e, owner);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int cc = lane + 32 * k;
      if (cc > jj && cc < bw) w[k] = __dsub_rn(w[k], __dmul_rn(e, __ldg(R + j * d + a + cc)));
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int cc = lane + 32 * k;
    if (cc < bw) codes[row * d + a + cc] = (uint8_t)q[k];
  }
}
