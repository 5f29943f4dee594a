// admmq.cu -- the ADMM-Q layer solve for B200 (sm_100a): setup kernels,
// packing, reductions, the tcgen05 GEMM instantiations and the C ABI
// declared in include/admmq.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cublas_v2.h>
#include <cusolverDn.h>

#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <type_traits>
#include <vector>

#include "../../include/admmq.h"
#include "kernels.cuh"
#include "admm_loop.cuh"

using namespace admmq;

namespace {

constexpr int kBM = 128;
unsigned long long g_launches = 0;  // kernels launched by this library
inline void count_launch() { __atomic_fetch_add(&g_launches, 1ull, __ATOMIC_RELAXED); }
// X^T X: bf16, both operands MN-major (X is token-major).  Promoted every 8
// k-blocks (32 MMAs of K = 16): measured 1226 TFLOP/s at q_proj against 1160
// with 4 k-blocks; 16 gained nothing more.
using GramCfg = GemmCfg<KIND_BF16, 1, true, true, 4, 8, false>;
// Eigenbasis GEMMs: K-major operands on CTA pairs (2-SM MMAs of 256 x 256
// tiles), 3 stages of 64 KB, promoted every KC k-blocks (K = 512 per chunk):
//   fp16 x3 (three full-rate fp16 products per K step, 96 MMAs per chunk):
//     the default for large layers;
//   mixed split (tf32 hi.hi + one bf16 product for the corrections, 128 MMAs
//     per chunk);
//   3xTF32 (three tf32 products, 192 MMAs per chunk): the default where the
//     reduction is short.
using EigCfg = GemmCfg<KIND_MIX, 2, false, false, 3, 16, true>;
using EigCfg3 = GemmCfg<KIND_TF32, 2, false, false, 3, 16, true>;
using EigCfgF = GemmCfg<KIND_F16X3, 2, false, false, 3, 8, true>;
static_assert(EigCfg::BN == EigCfg3::BN && EigCfg::BK == EigCfg3::BK && EigCfg::BN == EigCfgF::BN &&
                  EigCfg::UNIT_M == EigCfg3::UNIT_M && EigCfg::UNIT_M == EigCfgF::UNIT_M &&
                  EigCfg::B_ROWS == EigCfg3::B_ROWS && EigCfg::B_ROWS == EigCfgF::B_ROWS,
              "same tile geometry (K per stage differs: 32 fp32 or 64 fp16 elements)");
// d_in from which the automatic split mode picks the fp16 split
constexpr int kSplitFromDin = 2048;

// Setup status words (ws status[1]).
enum { SETUP_OK = 0, SETUP_NONFINITE = 1, SETUP_NOT_PD = 2 };

// ------------------------------------------------------------------ kernels

// sigma = Diag(H)^(-1/2), or 1 with scale == 0 (the unscaled ablation: the
// iteration then runs on H itself; diag H is still the refit's weight).
__global__ void k_diag_stats(const float* __restrict__ G, int d, float lambda_rel, int scale,
                             double* __restrict__ lam_out, double* __restrict__ sig64,
                             float* __restrict__ hdiag, float* __restrict__ sigma,
                             float* __restrict__ rsig, int* __restrict__ status) {
  __shared__ double red[1024];
  double acc = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) acc += (double)G[(long long)i * d + i];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  const double lam = (double)lambda_rel * red[0] / (double)d;
  if (threadIdx.x == 0) *lam_out = lam;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const double h = (double)G[(long long)i * d + i] + lam;
    if (!isfinite(h)) {
      atomicExch(&status[1], SETUP_NONFINITE);
    } else if (h <= 0.0) {
      atomicExch(&status[1], SETUP_NOT_PD);
    }
    const double sg = scale ? 1.0 / sqrt(h) : 1.0;
    sig64[i] = sg;
    hdiag[i] = (float)h;
    sigma[i] = (float)sg;
    rsig[i] = scale ? (float)sqrt(h) : 1.f;
  }
}

// H~ = Sigma (G + lambda I) Sigma in float64.
__global__ void k_scale_hessian(const float* __restrict__ G, int d, const double* __restrict__ lam,
                                const double* __restrict__ sig64, double* __restrict__ Ht) {
  const long long total = (long long)d * d;
  const double l = *lam;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx / d), j = (int)(idx - (long long)i * d);
    const double h = (double)G[idx] + (i == j ? l : 0.0);
    Ht[idx] = sig64[i] * h * sig64[j];
  }
}

template <typename T>
__device__ __forceinline__ float load_w(const T* p, long long i);
template <>
__device__ __forceinline__ float load_w<float>(const float* p, long long i) {
  return p[i];
}
template <>
__device__ __forceinline__ float load_w<__nv_bfloat16>(const __nv_bfloat16* p, long long i) {
  return __bfloat162float(p[i]);
}

#include "gptq.cuh"

// Power-of-two operand scale of each output row for the fp16 split.  Every
// A operand of the eigenbasis GEMMs is a row of the W~ family (W^~, P =
// D~ - V~, T, Delta~), whose entries stay within a small multiple of the
// row's norm ||W^~_j||; with 2^e_j ||W^~_j|| in [2^9, 2^10) they keep 64x
// headroom below fp16's largest value (an overflow raises the range flag)
// while the fp16 pair's absolute resolution stays far below what the
// row's products need.  row_out = 2^(-e_j - 14) undoes e_j and the B
// operands' 2^14 on a GEMM result.  Other encodings: 1 and 1.  One warp per
// row; the norm is summed in float64.
template <typename T>
__global__ void k_row_scales(const T* __restrict__ W, const float* __restrict__ rsig, int m, int d,
                             int enc, float* __restrict__ row_in, float* __restrict__ row_out) {
  const int warps = (int)(blockDim.x >> 5), lane = (int)(threadIdx.x & 31);
  for (long long row = blockIdx.x * (long long)warps + (threadIdx.x >> 5); row < m;
       row += (long long)gridDim.x * warps) {
    double n2 = 0.0;
    for (int i = lane; i < d; i += 32) {
      const double w = (double)__fmul_rn(load_w<T>(W, row * d + i), rsig[i]);
      n2 += w * w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
    if (lane == 0) {
      int e = 0;
      if (enc == ENC_F16) {
        const double nrm = sqrt(n2);
        if (nrm > 0.0 && isfinite(nrm)) {
          int k = 0;
          frexp(nrm, &k);  // nrm in [2^(k-1), 2^k)
          e = 10 - k;
          e = e < -60 ? -60 : (e > 60 ? 60 : e);
        }
        row_in[row] = ldexpf(1.f, e);
        row_out[row] = ldexpf(1.f, -e - kBScaleExp);
      } else {
        row_in[row] = 1.f;
        row_out[row] = 1.f;
      }
    }
  }
}

// W^~ = Sigma^-1 W_hat (rows = output channels) in the operand encoding (A side).
template <typename T>
__global__ void k_scale_weights(const T* __restrict__ W, const float* __restrict__ rsig, int d,
                                long long total, void* hi, void* lo, int enc,
                                const float* __restrict__ row_in, int* flag) {
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long row = idx / d;
    const int i = (int)(idx - row * d);
    const float w = __fmul_rn(load_w<T>(W, idx), rsig[i]);
    put_a1(enc, plane0_row(enc, hi, row, d), plane1_row(enc, lo, row, d), i, w, row_in[row], flag);
  }
}

// Eigenvector buffer (row k = k-th eigenvector, from the column-major solver
// output) -> operand planes (B side) of E = Q^T [k][i] and of Q [i][k]; the
// low part comes from the float64 value.
__global__ void k_split_eigvecs(const double* __restrict__ Evec, int d, void* e_hi, void* e_lo,
                                void* q_hi, void* q_lo, int enc) {
  __shared__ double tv[32][33];
  const int k0 = blockIdx.y * 32, i0 = blockIdx.x * 32;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int k = k0 + r, i = i0 + threadIdx.x;
    double e = 0.0;
    if (k < d && i < d) {
      e = Evec[(long long)k * d + i];
      put_b1(enc, plane0_row(enc, e_hi, k, d), plane1_row(enc, e_lo, k, d), i, e);
    }
    tv[r][threadIdx.x] = e;
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int i = i0 + r, k = k0 + threadIdx.x;
    if (k < d && i < d)
      put_b1(enc, plane0_row(enc, q_hi, i, d), plane1_row(enc, q_lo, i, d), k, tv[threadIdx.x][r]);
  }
}

__global__ void k_eigvals(const double* __restrict__ ev, int d, float* __restrict__ lam32,
                          int* __restrict__ status) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < d; i += gridDim.x * blockDim.x) {
    const double v = ev[i];
    if (!isfinite(v)) atomicExch(&status[2], 1);
    lam32[i] = (float)v;
  }
}

// RTN start: D_0 = min/max-grid rounding of W_hat, V~ = 0, P = D~_0 (operand
// encoding, A side).  One warp per (row, group): lane l takes the group's
// g/32 consecutive elements from l g/32 on, so the warp's accesses are
// contiguous; the group's min and max (exact in any order) come from a warp
// reduction and every lane forms the same grid from them.
template <typename T>
__global__ void k_init_rtn(const T* __restrict__ W, const float* __restrict__ rsig, int m, int d,
                           int g, int L, uint8_t* __restrict__ codes, float* __restrict__ scale,
                           float* __restrict__ zero, float* __restrict__ V, void* p_hi,
                           void* p_lo, int enc, const float* __restrict__ row_in, int* flag) {
  const int ngr = d / g, per = g / 32;
  const long long total = (long long)m * ngr;
  const float Lf = (float)L;
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long gi = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); gi < total;
       gi += warps) {
    const long long row = gi / ngr;
    const int col0 = (int)(gi - row * ngr) * g + lane * per;
    const long long base = row * d + col0;
    float y[4] = {0.f, 0.f, 0.f, 0.f};
    float mn = 0.f, mx = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e < per) {
        y[e] = load_w<T>(W, base + e);
        mn = fminf(mn, y[e]);
        mx = fmaxf(mx, y[e]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    float s = __fdiv_rn(__fsub_rn(mx, mn), Lf), z;
    if (s == 0.f) {
      s = 1.f;
      z = 0.f;
    } else {
      z = __fadd_rn(rintf(__fdiv_rn(-mn, s)), 0.f);
    }
    void* hi = plane0_row(enc, p_hi, row, d);
    void* lo = plane1_row(enc, p_lo, row, d);
    const float ri = row_in[row];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e >= per) break;
      const float q = clampq(__fadd_rn(rintf(__fdiv_rn(y[e], s)), z), Lf);
      const float D = __fmul_rn(s, __fsub_rn(q, z));
      const float dt = __fmul_rn(D, rsig[col0 + e]);
      codes[base + e] = (uint8_t)q;
      V[base + e] = 0.f;
      put_a1(enc, hi, lo, col0 + e, dt, ri, flag);
    }
    if (lane == 0) {
      scale[gi] = s;
      zero[gi] = z;
    }
  }
}

// Delta~ = D~ - W^~ (scaled coordinates) in the operand encoding (A side),
// for the objective.
template <typename T>
__global__ void k_delta_planes(const T* __restrict__ W, const uint8_t* __restrict__ codes,
                               const float* __restrict__ scale, const float* __restrict__ zero,
                               const float* __restrict__ rsig, int d, int g, long long total,
                               void* hi, void* lo, int enc, const float* __restrict__ row_in,
                               int* flag) {
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long row = idx / d;
    const int i = (int)(idx - row * d);
    const long long gi = row * (d / g) + i / g;
    const float D = __fmul_rn(scale[gi], __fsub_rn((float)codes[idx], zero[gi]));
    const float dt = __fmul_rn(D, rsig[i]);
    const float wt = __fmul_rn(load_w<T>(W, idx), rsig[i]);
    put_a1(enc, plane0_row(enc, hi, row, d), plane1_row(enc, lo, row, d), i, __fsub_rn(dt, wt),
           row_in[row], flag);
  }
}

// Fixed-order float64 reduction of per-tile partials.
__global__ void k_reduce_objective(const float* __restrict__ part, int count,
                                   double* __restrict__ out) {
  __shared__ double red[256];
  double acc = 0.0;
  for (int i = threadIdx.x; i < count; i += blockDim.x) acc += (double)part[i];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[0] = 0.5 * red[0];
}

__global__ void k_reduce_resid(const float* __restrict__ part, int per_iter, double rho0,
                               double gamma, double* __restrict__ out) {
  __shared__ double r2s[256], s2s[256];
  const int t = blockIdx.x;
  const float* p = part + (long long)t * per_iter * 2;
  double a = 0.0, b = 0.0;
  for (int i = threadIdx.x; i < per_iter; i += blockDim.x) {
    a += (double)p[2 * i];
    b += (double)p[2 * i + 1];
  }
  r2s[threadIdx.x] = a;
  s2s[threadIdx.x] = b;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) {
      r2s[threadIdx.x] += r2s[threadIdx.x + s];
      s2s[threadIdx.x] += s2s[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out[2 * t] = sqrt(r2s[0]);
    out[2 * t + 1] = rho0 * pow(gamma, (double)t) * sqrt(s2s[0]);
  }
}

// H = sum of the k-split partials over the upper triangle, mirrored; diagonal
// 32x32 blocks take every value from their upper half so H is symmetric.
__global__ void k_gram_finalize(const float* __restrict__ part, int splits, long long split_stride,
                                int d, float* __restrict__ H, int accumulate,
                                const int* __restrict__ status) {
  const int I = blockIdx.y, J = blockIdx.x;
  if (I > J) return;
  __shared__ float tile[32][33];
  const bool bad = status[0] != 0;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int i = I * 32 + r, j = J * 32 + threadIdx.x;
    float v = 0.f;
    if (i < d && j < d) {
      const long long off = (long long)i * d + j;
      for (int s = 0; s < splits; ++s) v += part[s * split_stride + off];
    }
    tile[r][threadIdx.x] = v;
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int c = threadIdx.x;
    // upper block (I, J): H[I*32 + r][J*32 + c]
    {
      const int i = I * 32 + r, j = J * 32 + c;
      if (i < d && j < d) {
        float v = (I == J && r > c) ? tile[c][r] : tile[r][c];
        if (bad && i == j) v = __int_as_float(0x7fc00000);
        const long long off = (long long)i * d + j;
        H[off] = accumulate ? H[off] + v : v;
      }
    }
    if (I != J) {  // mirrored block (J, I): H[J*32 + r][I*32 + c] = tile[c][r]
      const int i = J * 32 + r, j = I * 32 + c;
      if (i < d && j < d) {
        const long long off = (long long)i * d + j;
        H[off] = accumulate ? H[off] + tile[c][r] : tile[c][r];
      }
    }
  }
}

// Pack codes into a little-endian BITS-bit stream per row.  With d % 32 == 0
// the codes are a flat sequence of 32-code groups whose packed words (BITS
// per group) are contiguous as well, rows included.  A warp takes 32
// consecutive groups: lane l reads group l (32 bytes; the warp reads 1 KB
// contiguous), builds its BITS words, stages them in shared memory, and the
// warp writes its 32 x BITS words back as contiguous 16-byte stores.
template <int BITS>
__global__ void __launch_bounds__(256) k_pack(const uint8_t* __restrict__ codes, long long groups,
                                              uint32_t* __restrict__ out) {
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  __shared__ __align__(16) uint32_t stage[8][32 * BITS];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  uint32_t* buf = stage[wib];
  const long long nwarps = (long long)gridDim.x * 8;
  for (long long base = ((long long)blockIdx.x * 8 + wib) * 32; base < groups; base += nwarps * 32) {
    const long long grp = base + lane;
    uint32_t in[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (grp < groups) {
      const uint4* src = reinterpret_cast<const uint4*>(codes + grp * 32);
      const uint4 a = __ldcs(src), b = __ldcs(src + 1);
      in[0] = a.x; in[1] = a.y; in[2] = a.z; in[3] = a.w;
      in[4] = b.x; in[5] = b.y; in[6] = b.z; in[7] = b.w;
    }
    uint32_t w[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) w[k] = 0u;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const uint32_t v = (in[k >> 2] >> (8 * (k & 3))) & MASK;
      const int pos = k * BITS;
      w[pos >> 5] |= v << (pos & 31);
      if ((pos & 31) + BITS > 32) w[(pos >> 5) + 1] |= v >> (32 - (pos & 31));
    }
#pragma unroll
    for (int k = 0; k < BITS; ++k) buf[lane * BITS + k] = w[k];
    __syncwarp();
    const long long valid = groups - base < 32 ? groups - base : 32;
    uint32_t* dst = out + base * BITS;
    if (valid == 32) {
      // 32 * BITS words = 8 * BITS 16-byte vectors
      for (int v = lane; v < 8 * BITS; v += 32)
        __stcs(reinterpret_cast<uint4*>(dst) + v, reinterpret_cast<const uint4*>(buf)[v]);
    } else {
      for (int k = lane; k < valid * BITS; k += 32) dst[k] = buf[k];
    }
    __syncwarp();
  }
}

// rint_div8 on batches of eight values with one divisor per batch (tests).
__global__ void k_rint_div(const float* __restrict__ y, const float* __restrict__ s, long long batches,
                           float* __restrict__ out) {
  for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < batches;
       b += (long long)gridDim.x * blockDim.x) {
    float yy[8], q[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) yy[k] = y[8 * b + k];
    const float sb = s[b];
    rint_div8(yy, sb, __frcp_rn(sb), q);
#pragma unroll
    for (int k = 0; k < 8; ++k) out[8 * b + k] = q[k];
  }
}

// Standalone projection, W~ read from memory.  The passes over a group read
// each of its elements two or three times, and once enough warps run to
// cover the memory latency their groups (2 x g floats each) no longer stay
// in L1, so by default a block is one warp that first copies its rows' W~
// and V~ segments into shared memory (coalesced 16-byte asynchronous copies,
// a whole row segment per instruction for g = 128); the passes read them
// from there and DRAM sees each input once.  A lane takes one 32-column block
// of a (row, group): TPG = g / 32 lanes share a group and a warp holds 32 /
// TPG rows (8 for g = 128), so a warp stages about 11 KB whatever g is and
// many warps fit on an SM.  The rows' previous codes, scales and zero points
// are staged too, so the passes wait on no global load.  The 16-candidate
// error search of GRID_MSE is bound by arithmetic rather than memory, so it
// reads W~ and V~ from global memory (STAGED = false, 128-thread blocks, a
// thread per (row, group)).
__host__ __device__ constexpr int proj_rows(int tpg) { return 32 / tpg; }
// floats per row slot: W~ (g), V~ (g), 4 of padding so that the rows' 16-byte
// reads at one column spread over the banks; after the row slots, the
// group's sigma, 1/sigma and diag(H) (g each), shared by the block's rows;
// then the rows' previous codes (g + 16 bytes each) and their scales and zero
// points
__host__ __device__ constexpr int proj_slot(int g) { return 2 * g + 4; }
__host__ __device__ constexpr int proj_cols(int g, int tpg) { return proj_rows(tpg) * proj_slot(g); }
__host__ __device__ constexpr int proj_codes(int g, int tpg) { return proj_cols(g, tpg) + 3 * g; }
// a row's codes take g + 16 bytes, so the lanes of one 16-byte read phase
// (8 rows, the same column) fall on different banks
__host__ __device__ constexpr int proj_code_row(int g) { return g + 16; }
__host__ __device__ constexpr int proj_grid(int g, int tpg) {
  return proj_codes(g, tpg) + proj_rows(tpg) * proj_code_row(g) / 4;
}
__host__ __device__ constexpr int proj_floats(int g, int tpg) {
  return proj_grid(g, tpg) + 2 * proj_rows(tpg);
}

template <int MODE, int ENC, bool STAGED, int TPG>
__global__ void __launch_bounds__(STAGED ? 32 : 128) k_project(
    const float* __restrict__ wt, float* V, const float* __restrict__ sig,
    const float* __restrict__ rsig, const float* __restrict__ hd, int m, int d, int g, int L,
    uint8_t* codes, float* scale, float* zero, void* p_hi, void* p_lo,
    const float* __restrict__ row_in, int* flag, double* resid, float vs, int fit_w,
    int ahead) {
  static_assert(TPG == 1 || STAGED, "lanes that share a group share staged rows");
  constexpr int kRows = STAGED ? proj_rows(TPG) : 128;
  // staged launches have g = 32 TPG: a constant, so every index below folds
  if (STAGED) g = 32 * TPG;
  extern __shared__ float4 proj_smem[];
  float* stage = reinterpret_cast<float*>(proj_smem);
  const int lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRows;
  const int grp = blockIdx.y;
  const int col0 = grp * g;
  const int slot = proj_slot(g);
  if (STAGED) {
    // rows past m are filled with zeros (they are projected, never stored)
    const int per_row = g / 2;  // float4 pieces of W~ and V~ in one row
    const uint32_t sbase = smem_u32(stage);
#pragma unroll
    for (int i = lane; i < kRows * per_row; i += 32) {
      const int rr = i / per_row, piece = i - rr * per_row;
      const int arr = piece >= g / 4 ? 1 : 0;
      const int k = 4 * (piece - arr * (g / 4));
      const int off_s = rr * slot + arr * g + k;
      if (row0 + rr < m) {
        const float* src = (arr ? V : wt) + (long long)(row0 + rr) * d + col0 + k;
        cp_async16(sbase + 4u * (uint32_t)off_s, src);
      } else {
        *reinterpret_cast<float4*>(stage + off_s) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float* cols = stage + kRows * slot;
#pragma unroll
    for (int i = lane; i < 3 * (g / 4); i += 32) {
      const int v = i / (g / 4), k = 4 * (i - v * (g / 4));
      const float* src = (v == 0 ? sig : v == 1 ? rsig : hd) + col0 + k;
      cp_async16(smem_u32(cols + v * g + k), src);
    }
    // the previous codes of this block's rows and their scale and zero point
    uint8_t* cs = reinterpret_cast<uint8_t*>(stage + proj_codes(g, TPG));
#pragma unroll
    for (int i = lane; i < kRows * (g / 16); i += 32) {
      const int rr = i / (g / 16), k = 16 * (i - rr * (g / 16));
      if (row0 + rr < m)
        cp_async16(smem_u32(cs + rr * proj_code_row(g) + k),
                   codes + (long long)(row0 + rr) * d + col0 + k);
    }
    float* gs = stage + proj_grid(g, TPG);
    if (lane < kRows && row0 + lane < m) {
      const long long gi = (long long)(row0 + lane) * (d / g) + grp;
      cp_async4(smem_u32(gs + lane), scale + gi);
      cp_async4(smem_u32(gs + kRows + lane), zero + gi);
    }
    // Blocks start in the order of their linear index, so the block `ahead`
    // (one resident wave) later will run on an SM about when this one ends:
    // bring its rows into L2 now, so that its copies find them there.
    if (ahead > 0) {  // the grid has fewer than 2^31 blocks (the host checks)
      const unsigned lin = blockIdx.x + blockIdx.y * gridDim.x + (unsigned)ahead;
      if (lin < gridDim.x * gridDim.y) {
        const int r0 = (int)(lin % gridDim.x) * kRows, c0 = (int)(lin / gridDim.x) * g;
        if (lane < kRows && r0 + lane < m) {
          const long long o = (long long)(r0 + lane) * d + c0;
          prefetch_l2_bulk(wt + o, 4u * (uint32_t)g);
          prefetch_l2_bulk(V + o, 4u * (uint32_t)g);
          prefetch_l2_bulk(codes + o, (uint32_t)g);
        }
      }
    }
    cp_async_wait_all();
    __syncwarp();
  }
  // this thread's row of the block and its 32-column block of the group
  const int rr = TPG > 1 ? lane % kRows : (int)threadIdx.x;
  const int blk = TPG > 1 ? lane / kRows : 0;
  const int hc = 32 * blk;  // first column of this thread within the group
  const int row = row0 + rr;
  const bool valid = row < m;
  const long long off = (long long)(valid ? row : 0) * d + col0 + hc;
  const long long goff = (long long)(valid ? row : 0) * (d / g) + grp;
  ProjRow r;
  r.V = V + off;
  if (STAGED) {
    const float* cols = stage + kRows * slot;
    r.sig = cols + hc;
    r.rsig = cols + g + hc;
    r.hd = cols + 2 * g + hc;
  } else {
    r.sig = sig + col0;
    r.rsig = rsig + col0;
    r.hd = hd + col0;
  }
  r.codes = codes + off;
  r.phi = plane0_at(ENC, p_hi, valid ? row : 0, d, col0 + hc);
  r.plo = plane1_at(ENC, p_lo, valid ? row : 0, d, col0 + hc);
  r.scale = scale + goff;
  r.zero = zero + goff;
  r.wdump = nullptr;
  r.rs = (valid && row_in) ? row_in[row] : 1.f;
  r.vs = vs;
  r.fit_w = fit_w;
  r.flag = flag;
  r.valid = valid;
  r.grid_out = blk == 0;
  if (STAGED) {
    r.codes_in = reinterpret_cast<const uint8_t*>(stage + proj_codes(g, TPG)) + rr * proj_code_row(g) + hc;
    r.scale_in = stage + proj_grid(g, TPG) + rr;
    r.zero_in = stage + proj_grid(g, TPG) + kRows + rr;
  } else {
    r.codes_in = nullptr;
    r.scale_in = nullptr;
    r.zero_in = nullptr;
  }
  const float* mine = stage + rr * slot + hc;
  auto loadw = [&](int c, float (&w)[32]) {
#pragma unroll
    for (int k = 0; k < 32; k += 4) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (STAGED)
        v = *reinterpret_cast<const float4*>(mine + c + k);
      else if (valid)
        v = *reinterpret_cast<const float4*>(wt + off + c + k);
      w[k] = v.x; w[k + 1] = v.y; w[k + 2] = v.z; w[k + 3] = v.w;
    }
  };
  auto loadv = [&](int c, float (&v)[8]) {
    if (STAGED) {
      const float4 a = *reinterpret_cast<const float4*>(mine + g + c);
      const float4 b = *reinterpret_cast<const float4*>(mine + g + c + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else if (valid) {
      ld_v8f(r.V + c, v);
    }
  };
  float r2 = 0.f, s2 = 0.f;
  project_group<MODE, ENC, STAGED, TPG>(loadw, loadv, r, g, L, r2, s2);
  r2 = warp_sum(r2);
  s2 = warp_sum(s2);
  if (lane == 0) {
    atomicAdd(&resid[0], (double)r2);
    atomicAdd(&resid[1], (double)s2);
  }
}

// ------------------------------------------------------------- host utils

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Row-major [outer][inner] tensor of fp32, bf16 or fp16, box {128 bytes,
// box_outer}, 128-byte swizzle, out-of-bounds elements read as zero.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer,
              CUtensorMapDataType dt) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint32_t es = dt == CU_TENSOR_MAP_DATA_TYPE_FLOAT32 ? 4 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * es};
  cuuint32_t box[2] = {128 / es, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The two planes of an operand [rows][d] in encoding `enc` (see kernels.cuh).
bool make_plane_maps(CUtensorMap (&mp)[2], void* hi, void* lo, uint64_t d, uint64_t rows,
                     uint32_t box_rows, int enc) {
  if (enc == ENC_F16)
    return make_map(&mp[0], hi, d, rows, box_rows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) &&
           make_map(&mp[1], lo, d, rows, box_rows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  if (enc == ENC_MIX)
    return make_map(&mp[0], hi, d, rows, box_rows, CU_TENSOR_MAP_DATA_TYPE_FLOAT32) &&
           make_map(&mp[1], lo, 2 * d, rows, box_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  return make_map(&mp[0], hi, d, rows, box_rows, CU_TENSOR_MAP_DATA_TYPE_FLOAT32) &&
         make_map(&mp[1], lo, d, rows, box_rows, CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
}

int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

// 128-row x BN tiles of an eigenbasis GEMM output [m][d] (per-tile partials)
int eig_tiles(int m, int d) {
  return cdiv(m, EigCfg::UNIT_M) * (EigCfg::UNIT_M / kBM) * cdiv(d, 128);
}

GemmGeom make_geom(int M, int N, long long K, int BN, int BK, int splits, bool triangle,
                   int* status, int unit_m = kBM) {
  GemmGeom g;
  g.M = M;
  g.N = N;
  g.K = (int)K;
  // 128-row tiles, counted up to whole units (a CTA pair's second tile may
  // lie past M: its epilogue masks every row, its partial sums are zeros)
  g.tiles_mu = cdiv(M, unit_m);
  g.tiles_m = g.tiles_mu * (unit_m / kBM);
  g.tiles_n = cdiv(N, BN);
  g.kblocks = cdiv(K, BK);
  g.splits = splits;
  g.triangle = triangle ? 1 : 0;
  if (!triangle) {
    g.tiles = g.tiles_mu * g.tiles_n;
  } else {
    int t = 0;
    for (int tn = 0; tn < g.tiles_n; ++tn) {
      int cnt = cdiv((long long)(tn + 1) * BN, kBM);
      t += cnt < g.tiles_m ? cnt : g.tiles_m;
    }
    g.tiles = t;
  }
  g.units = g.tiles * splits;
  // bands of 8 unit rows: measured best of 4, 8, 12, 16 for the eigenbasis
  // GEMMs at q_proj (ms per solve 75.0, 73.8, 75.3, 79.7)
  g.band = g.tiles_mu < 8 ? g.tiles_mu : 8;
  g.status = status;
  return g;
}

// Geometry of an eigenbasis GEMM [rows][d] x [d][d] for an encoding (its K
// per stage: 32 fp32 or 64 fp16 elements).  A band's A panels (band unit
// rows x d x the encoding's bytes per element, both planes) are re-read for
// every tile column of the band, so they should stay in L2: the band is the
// most unit rows (at most 8) whose panels fit 48 MiB.  Measured per fused
// launch at d = 12288 (down_proj, fp16 split, 12.6 MB of A per unit row):
// bands 2 / 3 / 4 / 5 / 6 / 8 took 612-619 / 602-604 / 598-599 / 602 /
// 599-604 / 615-616 ms; at d = 4096 (4 MB per unit row) bands 4-12 are
// within 1% and 8 is kept.
GemmGeom eig_geom(int enc, int rows, int d, int* status) {
  GemmGeom g = enc == ENC_F16
                   ? make_geom(rows, d, d, EigCfgF::BN, EigCfgF::BK, 1, false, status, EigCfgF::UNIT_M)
                   : make_geom(rows, d, d, EigCfg::BN, EigCfg::BK, 1, false, status, EigCfg::UNIT_M);
  const long long unit_m = enc == ENC_F16 ? EigCfgF::UNIT_M : EigCfg::UNIT_M;
  const long long elem = enc == ENC_F16 ? 4 : 8;  // bytes per A element over both planes
  const long long fit = (48ll << 20) / (unit_m * (long long)d * elem);
  const int cap = fit < 1 ? 1 : (fit > 8 ? 8 : (int)fit);
  if (g.band > cap) g.band = cap;
  return g;
}

// Launches k_gemm<Cfg, Work> over `units` work units: one CTA per SM, or one
// pair of CTAs per two SMs.  A policy whose units wait on earlier units of the
// same launch deals them from a counter to the CTAs that are running, so it
// needs none resident in particular; its grid is the occupancy query's count,
// the most CTAs that can run at once.
template <class Cfg, class Work>
cudaError_t launch_work(const typename Work::Args& args, int units, cudaStream_t st) {
  auto kern = k_gemm<Cfg, Work>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) return e;
  if (units <= 0) return cudaSuccess;
  if (!Cfg::PAIR) {
    int grid = num_sms();
    if (Work::SIGNALS) {
      int per_sm = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Cfg::THREADS, Cfg::SMEM);
      if (e != cudaSuccess) return e;
      if (per_sm < 1) return cudaErrorInvalidConfiguration;
      grid = per_sm * num_sms();
    }
    if (units < grid) grid = units;
    count_launch();
    kern<<<grid, Cfg::THREADS, Cfg::SMEM, st>>>(args);
    return cudaGetLastError();
  }
  // CTA pairs: clusters of two, one work unit per cluster at a time
  int pairs = num_sms() / 2;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2 * pairs);
  lc.blockDim = dim3(Cfg::THREADS);
  lc.dynamicSmemBytes = Cfg::SMEM;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  if (Work::SIGNALS) {
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &lc);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    if (clusters < pairs) pairs = clusters;
  }
  lc.gridDim = dim3(2 * (units < pairs ? units : pairs));
  count_launch();
  e = cudaLaunchKernelEx(&lc, kern, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <class Cfg, class Epi>
cudaError_t launch_gemm(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b0,
                        const CUtensorMap& b1, const GemmGeom& g, const typename Epi::Params& ep,
                        cudaStream_t st) {
  typename OneGemm<Epi>::Args x;
  x.a[0] = a0;
  x.a[1] = a1;
  x.b[0] = b0;
  x.b[1] = b1;
  x.g = g;
  x.ep = ep;
  return launch_work<Cfg, OneGemm<Epi>>(x, g.units, st);
}

// An eigenbasis GEMM (A and B operand maps, plane 0 and 1) with the split
// precision of the context: Epi3 for 3xTF32, EpiM for the mixed split, EpiF
// for the fp16 split.
template <class Epi3, class EpiM, class EpiF>
cudaError_t launch_eig(int enc, const CUtensorMap (&a)[2], const CUtensorMap (&b)[2],
                       const GemmGeom& g, const typename EpiM::Params& ep, cudaStream_t st) {
  static_assert(std::is_same<typename Epi3::Params, typename EpiM::Params>::value &&
                    std::is_same<typename EpiF::Params, typename EpiM::Params>::value,
                "same params");
  if (enc == ENC_F16) return launch_gemm<EigCfgF, EpiF>(a[0], a[1], b[0], b[1], g, ep, st);
  if (enc == ENC_MIX) return launch_gemm<EigCfg, EpiM>(a[0], a[1], b[0], b[1], g, ep, st);
  return launch_gemm<EigCfg3, Epi3>(a[0], a[1], b[0], b[1], g, ep, st);
}

int device_ok() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ADMMQ_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return ADMMQ_ERR_CUDA;
  return major == 10 ? ADMMQ_OK : ADMMQ_ERR_UNSUPPORTED;
}

int grid_for(long long work, int per_block = 256) {
  long long b = (work + per_block - 1) / per_block;
  long long cap = (long long)num_sms() * 8;
  if (b > cap) b = cap;
  return b < 1 ? 1 : (int)b;
}

// Gram k-split count: the smallest split (1..8) whose units fill the SMs best.
int gram_splits(long long n, int d, int nsm) {
  GemmGeom g = make_geom(d, d, n, GramCfg::BN, GramCfg::BK, 1, true, nullptr);
  int best = 1;
  double best_eff = -1.0;
  for (int s = 1; s <= 8; ++s) {
    if (s > g.kblocks) break;
    long long units = (long long)g.tiles * s;
    long long waves = (units + nsm - 1) / nsm;
    double eff = (double)units / (double)(waves * nsm);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
bool aligned32(const void* p) { return ((uintptr_t)p & 31) == 0; }

}  // namespace

// =================================================================== C ABI

struct admmq_ctx {
  int d, m, L, dev;
  admmq_params p;
  uint8_t* ws;
  size_t ws_bytes;
  int* status;          // [4]
  double* lam64;        // damping lambda
  double* sig64;        // [d]
  float *hdiag, *sigma, *rsig, *lam32;
  double* Ht;           // [d][d]  H~, then eigenvectors (row k = eigenvector k)
  double* evals;        // [d]
  double* work;
  int lwork;
  int* devinfo;
  // operand planes in the encoding `enc` (ENC_*, kernels.cuh): A side Wt, P,
  // T [m][d]; B side E, Q [d][d]
  int enc;
  void *E_hi, *Q_hi;
  void *E_lo, *Q_lo;
  void *Wt_hi, *P_hi, *T_hi;
  void *Wt_lo, *P_lo, *T_lo;
  float *row_in, *row_out;  // [m] per-row operand scale and result factor (fp16 split)
  float *C0, *V;                               // [m][d]
  float* resid_part;    // [iters][tiles][4][2]
  float* obj_part;      // [tiles][4]
  float* rho_tab;       // [iters] rho_t, as the host computes it
  float* vscale_tab;    // [iters] the dual's factor after iteration t (1 without rescaling)
  int* ready;           // [2][unit rows] ready counters of the fused schedule
  int ready_base;       // iterations counted in `ready` since admmq_init zeroed it
  int* ticket;          // [2] unit tickets of the fused launches, used alternately
  unsigned fused_launches;  // fused launches since admmq_init
  int tiles_eig;
  const void* W_hat;
  int w_dtype;
  float* wdump;
  cusolverDnHandle_t solver;
  CUtensorMap mWt[2], mP[2], mT[2], mE[2], mQ[2];
  bool timing;
  struct TimingRec {
    cudaEvent_t a, b, c;  // GEMM 1 = a..b, GEMM 2 = b..c; fused: a..b, c unused
    bool fused;
    int iters;
  };
  std::vector<TimingRec> ev;
  bool prepared, eig_done, inited;
};

namespace {

struct Layout {
  size_t status, lam64, sig64, hdiag, sigma, rsig, lam32, Ht, evals, work, devinfo;
  size_t E_hi, E_lo, Q_hi, Q_lo, Wt_hi, Wt_lo, P_hi, P_lo, T_hi, T_lo, C0, V;
  size_t resid_part, obj_part, rho_tab, ready, row_in, row_out, total;
};

Layout make_layout(int d, int m, int iters, int lwork) {
  Layout L;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  const size_t dd = (size_t)d * d, md = (size_t)m * d;
  const int tiles = eig_tiles(m, d);
  L.status = take(16);
  L.lam64 = take(8);
  L.sig64 = take(8 * (size_t)d);
  L.hdiag = take(4 * (size_t)d);
  L.sigma = take(4 * (size_t)d);
  L.rsig = take(4 * (size_t)d);
  L.lam32 = take(4 * (size_t)d);
  L.Ht = take(8 * dd);
  L.evals = take(8 * (size_t)d);
  L.work = take(8 * (size_t)(lwork > 0 ? lwork : 1));
  L.devinfo = take(16);
  L.E_hi = take(4 * dd);
  L.E_lo = take(4 * dd);
  L.Q_hi = take(4 * dd);
  L.Q_lo = take(4 * dd);
  L.Wt_hi = take(4 * md);
  L.Wt_lo = take(4 * md);
  L.P_hi = take(4 * md);
  L.P_lo = take(4 * md);
  L.T_hi = take(4 * md);
  L.T_lo = take(4 * md);
  L.C0 = take(4 * md);
  L.V = take(4 * md);
  L.resid_part = take(4 * (size_t)(iters > 0 ? iters : 1) * tiles * 8);
  L.obj_part = take(4 * (size_t)tiles * 4);
  L.rho_tab = take(4 * 2 * (size_t)(iters > 0 ? iters : 1));  // rho_t, then the dual factors
  L.ready = take(4 * (2 * (size_t)cdiv(m, 2 * kBM) + 2));  // counters, then 2 tickets
  L.row_in = take(4 * (size_t)m);
  L.row_out = take(4 * (size_t)m);
  L.total = o;
  return L;
}

void destroy_events(admmq_ctx* c) {
  for (auto& r : c->ev) {
    if (r.a) cudaEventDestroy(r.a);
    if (r.b) cudaEventDestroy(r.b);
    if (r.c) cudaEventDestroy(r.c);
  }
  c->ev.clear();
}

// rho_t = rho0 gamma^t, evaluated in double and rounded once to float.
float rho_at(const admmq_params& p, int t) {
  return (float)((double)p.rho0 * pow((double)p.gamma, (double)t));
}

// Factor applied to V~ after iteration t: rho_t / rho_{t+1} (evaluated in
// double, rounded once) with params.rescale_dual, else exactly 1.
float vscale_at(const admmq_params& p, int t) {
  if (!p.rescale_dual) return 1.f;
  const double a = (double)p.rho0 * pow((double)p.gamma, (double)t);
  const double b = (double)p.rho0 * pow((double)p.gamma, (double)(t + 1));
  return (float)(a / b);
}

int check_params(int d, int m, const admmq_params* p) {
  if (!p) return ADMMQ_ERR_INVALID_ARG;
  if (d <= 0 || m <= 0 || d % 32 != 0) return ADMMQ_ERR_INVALID_ARG;
  if (!(p->group == 32 || p->group == 64 || p->group == 128) || d % p->group != 0)
    return ADMMQ_ERR_INVALID_ARG;
  if (p->bits < 1 || p->bits > 8 || p->iters < 0) return ADMMQ_ERR_INVALID_ARG;
  if (!(p->rho0 > 0.f) || !(p->gamma > 0.f) || !(p->lambda_rel >= 0.f)) return ADMMQ_ERR_INVALID_ARG;
  if (p->grid_mode < ADMMQ_GRID_MINMAX || p->grid_mode > ADMMQ_GRID_MSE)
    return ADMMQ_ERR_INVALID_ARG;
  if (p->split_mode < ADMMQ_SPLIT_AUTO || p->split_mode > ADMMQ_SPLIT_F16)
    return ADMMQ_ERR_INVALID_ARG;
  if (p->no_scaling != 0 && p->no_scaling != 1) return ADMMQ_ERR_INVALID_ARG;
  if (p->rescale_dual != 0 && p->rescale_dual != 1) return ADMMQ_ERR_INVALID_ARG;
  if (p->fit_on_w != 0 && p->fit_on_w != 1) return ADMMQ_ERR_INVALID_ARG;
  if (p->schedule != ADMMQ_SCHEDULE_FUSED && p->schedule != ADMMQ_SCHEDULE_PER_GEMM)
    return ADMMQ_ERR_INVALID_ARG;
  return ADMMQ_OK;
}

int syevd_lwork(int d) {
  static cusolverDnHandle_t h = nullptr;
  if (!h && cusolverDnCreate(&h) != CUSOLVER_STATUS_SUCCESS) return -1;
  int lwork = 0;
  if (cusolverDnDsyevd_bufferSize(h, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_UPPER, d, nullptr,
                                  d, nullptr, &lwork) != CUSOLVER_STATUS_SUCCESS)
    return -1;
  return lwork;
}

// ------------------------------------------------------------ GPTQ host side

// Library handles for the GPTQ baseline (created on first use, for the
// device current at that time).
cusolverDnHandle_t gptq_solver() {
  static cusolverDnHandle_t h = nullptr;
  if (!h && cusolverDnCreate(&h) != CUSOLVER_STATUS_SUCCESS) h = nullptr;
  return h;
}
cublasHandle_t gptq_blas() {
  static cublasHandle_t h = nullptr;
  if (!h && cublasCreate(&h) != CUBLAS_STATUS_SUCCESS) h = nullptr;
  return h;
}

int gptq_lwork(int d) {
  cusolverDnHandle_t h = gptq_solver();
  if (!h) return -1;
  int l1 = 0, l2 = 0;
  if (cusolverDnDpotrf_bufferSize(h, CUBLAS_FILL_MODE_LOWER, d, nullptr, d, &l1) !=
          CUSOLVER_STATUS_SUCCESS ||
      cusolverDnDpotri_bufferSize(h, CUBLAS_FILL_MODE_LOWER, d, nullptr, d, &l2) !=
          CUSOLVER_STATUS_SUCCESS)
    return -1;
  return l1 > l2 ? l1 : l2;
}

// GPTQ workspace: status words, lambda and the damping kernel's per-column
// outputs, H in float64 (factorised in place into R), the float64 working
// weights, one block of errors E, the solver's work area.
struct GptqLayout {
  size_t status, lam64, sig64, hdiag, sigma, rsig, Hd, Wd, E, work, devinfo, total;
};

GptqLayout gptq_layout(int d, int m, int block, int lwork) {
  GptqLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.status = take(16);
  L.lam64 = take(8);
  L.sig64 = take(8 * (size_t)d);
  L.hdiag = take(4 * (size_t)d);
  L.sigma = take(4 * (size_t)d);
  L.rsig = take(4 * (size_t)d);
  L.Hd = take(8 * (size_t)d * d);
  L.Wd = take(8 * (size_t)d * m);
  L.E = take(8 * (size_t)m * block);
  L.work = take(8 * (size_t)(lwork > 0 ? lwork : 1));
  L.devinfo = take(16);
  L.total = o;
  return L;
}

#define CK(x)                                      \
  do {                                             \
    if ((x) != cudaSuccess) return ADMMQ_ERR_CUDA; \
  } while (0)

// GEMM 1 and GEMM 2 of iterations t0 .. t0+count-1 in one launch.
template <class Cfg, class E1, class E2>
cudaError_t launch_admm_loop(const admmq_ctx* c, const GemmGeom& g, const TUpdateParams& p1,
                             const ProjParams& p2, int t0, int count, cudaStream_t st) {
  using W = AdmmLoop<E1, E2>;
  typename W::Args x;
  for (int p = 0; p < 2; ++p) {
    x.a[0][p] = c->mP[p];
    x.b[0][p] = c->mE[p];
    x.a[1][p] = c->mT[p];
    x.b[1][p] = c->mQ[p];
  }
  x.g = g;
  x.p1 = p1;
  x.p2 = p2;
  x.rho = c->rho_tab;
  x.vscale = c->vscale_tab;
  x.part0 = c->resid_part;
  x.part_stride = (long long)c->tiles_eig * 8;
  x.ready = c->ready;
  x.base = c->ready_base;
  x.ticket = c->ticket + (c->fused_launches & 1u);
  x.ticket_next = c->ticket + ((c->fused_launches + 1u) & 1u);
  x.ctas = Cfg::PAIR ? 2 : 1;
  x.t0 = t0;
  x.count = count;
  return launch_work<Cfg, W>(x, count * 2 * g.units, st);
}

template <int MODE>
cudaError_t launch_admm_loop_split(const admmq_ctx* c, const GemmGeom& g, const TUpdateParams& p1,
                                   const ProjParams& p2, int t0, int count, cudaStream_t st) {
  if (c->enc == ENC_F16)
    return launch_admm_loop<EigCfgF, EpiTUpdate<ENC_F16>, EpiProject<MODE, ENC_F16>>(c, g, p1, p2, t0,
                                                                                     count, st);
  if (c->enc == ENC_MIX)
    return launch_admm_loop<EigCfg, EpiTUpdate<ENC_MIX>, EpiProject<MODE, ENC_MIX>>(c, g, p1, p2, t0,
                                                                                    count, st);
  return launch_admm_loop<EigCfg3, EpiTUpdate<ENC_TF32X3>, EpiProject<MODE, ENC_TF32X3>>(c, g, p1, p2,
                                                                                         t0, count, st);
}

}  // namespace

extern "C" {

const char* admmq_status_string(int s) {
  switch (s) {
    case ADMMQ_OK: return "ok";
    case ADMMQ_ERR_INVALID_ARG: return "invalid argument";
    case ADMMQ_ERR_CUDA: return "CUDA error";
    case ADMMQ_ERR_EIG: return "eigensolver failed";
    case ADMMQ_ERR_NOT_PD: return "Hessian diagonal not positive";
    case ADMMQ_ERR_NONFINITE: return "non-finite value in the Hessian or its eigenvalues";
    case ADMMQ_ERR_TIMEOUT: return "kernel pipeline wait timed out";
    case ADMMQ_ERR_WORKSPACE: return "workspace too small";
    case ADMMQ_ERR_UNSUPPORTED: return "unsupported device or shape";
    case ADMMQ_ERR_RANGE: return "an fp16-split operand left fp16's range";
    default: return "unknown status";
  }
}

int admmq_version(void) { return 102; }

int64_t admmq_launch_count(void) { return (int64_t)__atomic_load_n(&g_launches, __ATOMIC_RELAXED); }

size_t admmq_gram_workspace_bytes(int64_t n, int d_in) {
  if (d_in <= 0 || d_in % 32 != 0 || n < 0) return 0;
  const int s = gram_splits(n > 0 ? n : 1, d_in, num_sms());
  return 256 + (size_t)s * d_in * d_in * 4;
}

int admmq_build_hessian(const void* X, int64_t n, int d, float* H, int accumulate, void* ws,
                        size_t ws_bytes, void* stream) {
  if ((!X && n > 0) || !H || d <= 0 || d % 32 != 0 || n < 0 || !ws) return ADMMQ_ERR_INVALID_ARG;
  if (((uintptr_t)X & 15) != 0) return ADMMQ_ERR_INVALID_ARG;
  int rc = device_ok();
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t dd4 = (size_t)d * d * 4;
  if (ws_bytes < 256 + dd4) return ADMMQ_ERR_WORKSPACE;
  if (n == 0) {
    if (!accumulate) CK(cudaMemsetAsync(H, 0, dd4, st));
    return ADMMQ_OK;
  }
  int splits = gram_splits(n, d, num_sms());
  while (splits > 1 && ws_bytes < 256 + (size_t)splits * dd4) --splits;
  int* status = (int*)ws;
  float* part = (float*)((uint8_t*)ws + 256);
  CK(cudaMemsetAsync(status, 0, 16, st));
  CUtensorMap mx;
  if (!make_map(&mx, X, (uint64_t)d, (uint64_t)n, GramCfg::BK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) return ADMMQ_ERR_CUDA;
  GemmGeom g = make_geom(d, d, n, GramCfg::BN, GramCfg::BK, splits, true, status);
  EpiGramPartial::Params ep{part, (long long)d * d, d};
  CK((launch_gemm<GramCfg, EpiGramPartial>(mx, mx, mx, mx, g, ep, st)));
  const int nb = d / 32;
  count_launch(), k_gram_finalize<<<dim3(nb, nb), dim3(32, 8), 0, st>>>(part, splits, (long long)d * d, d, H,
                                                        accumulate, status);
  CK(cudaGetLastError());
  return ADMMQ_OK;
}

size_t admmq_workspace_bytes(int d_in, int d_out, const admmq_params* p) {
  if (check_params(d_in, d_out, p)) return 0;
  const int lwork = syevd_lwork(d_in);
  if (lwork < 0) return 0;
  return make_layout(d_in, d_out, p->iters, lwork).total;
}

int admmq_create(admmq_ctx** out, int d, int m, const admmq_params* p, void* ws, size_t ws_bytes) {
  if (!out) return ADMMQ_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = check_params(d, m, p);
  if (rc) return rc;
  if (!ws || ((uintptr_t)ws & 255) != 0) return ADMMQ_ERR_INVALID_ARG;
  rc = device_ok();
  if (rc) return rc;
  const int lwork = syevd_lwork(d);
  if (lwork < 0) return ADMMQ_ERR_EIG;
  Layout L = make_layout(d, m, p->iters, lwork);
  if (ws_bytes < L.total) return ADMMQ_ERR_WORKSPACE;
  admmq_ctx* c = new admmq_ctx();
  c->d = d;
  c->m = m;
  c->p = *p;
  c->L = (1 << p->bits) - 1;
  c->enc = p->split_mode == ADMMQ_SPLIT_MIXED    ? ENC_MIX
           : p->split_mode == ADMMQ_SPLIT_3XTF32 ? ENC_TF32X3
           : p->split_mode == ADMMQ_SPLIT_F16    ? ENC_F16
           : (d >= kSplitFromDin ? ENC_F16 : ENC_TF32X3);
  cudaGetDevice(&c->dev);
  c->ws = (uint8_t*)ws;
  c->ws_bytes = ws_bytes;
  uint8_t* b = c->ws;
  c->status = (int*)(b + L.status);
  c->lam64 = (double*)(b + L.lam64);
  c->sig64 = (double*)(b + L.sig64);
  c->hdiag = (float*)(b + L.hdiag);
  c->sigma = (float*)(b + L.sigma);
  c->rsig = (float*)(b + L.rsig);
  c->lam32 = (float*)(b + L.lam32);
  c->Ht = (double*)(b + L.Ht);
  c->evals = (double*)(b + L.evals);
  c->work = (double*)(b + L.work);
  c->lwork = lwork;
  c->devinfo = (int*)(b + L.devinfo);
  c->E_hi = (void*)(b + L.E_hi);
  c->E_lo = (void*)(b + L.E_lo);
  c->Q_hi = (void*)(b + L.Q_hi);
  c->Q_lo = (void*)(b + L.Q_lo);
  c->Wt_hi = (void*)(b + L.Wt_hi);
  c->Wt_lo = (void*)(b + L.Wt_lo);
  c->P_hi = (void*)(b + L.P_hi);
  c->P_lo = (void*)(b + L.P_lo);
  c->T_hi = (void*)(b + L.T_hi);
  c->T_lo = (void*)(b + L.T_lo);
  c->C0 = (float*)(b + L.C0);
  c->V = (float*)(b + L.V);
  c->resid_part = (float*)(b + L.resid_part);
  c->obj_part = (float*)(b + L.obj_part);
  c->rho_tab = (float*)(b + L.rho_tab);
  c->vscale_tab = c->rho_tab + (p->iters > 0 ? p->iters : 1);
  c->ready = (int*)(b + L.ready);
  c->ticket = c->ready + 2 * cdiv(m, 2 * kBM);
  c->tiles_eig = eig_tiles(m, d);
  bool ok = true;
  c->row_in = (float*)(b + L.row_in);
  c->row_out = (float*)(b + L.row_out);
  ok &= make_plane_maps(c->mWt, c->Wt_hi, c->Wt_lo, d, m, kBM, c->enc);
  ok &= make_plane_maps(c->mP, c->P_hi, c->P_lo, d, m, kBM, c->enc);
  ok &= make_plane_maps(c->mT, c->T_hi, c->T_lo, d, m, kBM, c->enc);
  ok &= make_plane_maps(c->mE, c->E_hi, c->E_lo, d, d, EigCfg::B_ROWS, c->enc);
  ok &= make_plane_maps(c->mQ, c->Q_hi, c->Q_lo, d, d, EigCfg::B_ROWS, c->enc);
  if (!ok || cusolverDnCreate(&c->solver) != CUSOLVER_STATUS_SUCCESS) {
    delete c;
    return ADMMQ_ERR_CUDA;
  }
  *out = c;
  return ADMMQ_OK;
}

void admmq_destroy(admmq_ctx* c) {
  if (!c) return;
  destroy_events(c);
  if (c->solver) cusolverDnDestroy(c->solver);
  delete c;
}

int admmq_prepare(admmq_ctx* c, const float* G, const void* W_hat, int w_dtype, void* stream) {
  if (!c || !G || !W_hat) return ADMMQ_ERR_INVALID_ARG;
  if (w_dtype != ADMMQ_DTYPE_F32 && w_dtype != ADMMQ_DTYPE_BF16) return ADMMQ_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int d = c->d, m = c->m;
  c->W_hat = W_hat;
  c->w_dtype = w_dtype;
  CK(cudaMemsetAsync(c->status, 0, 16, st));
  count_launch(), k_diag_stats<<<1, 1024, 0, st>>>(G, d, c->p.lambda_rel, !c->p.no_scaling, c->lam64, c->sig64, c->hdiag, c->sigma,
                                   c->rsig, c->status);
  CK(cudaGetLastError());
  count_launch(), k_scale_hessian<<<grid_for((long long)d * d), 256, 0, st>>>(G, d, c->lam64, c->sig64, c->Ht);
  CK(cudaGetLastError());
  const long long md = (long long)m * d;
  int* flag = c->status + 3;
  if (w_dtype == ADMMQ_DTYPE_F32) {
    count_launch(), k_row_scales<float><<<grid_for(m, 8), 256, 0, st>>>((const float*)W_hat, c->rsig, m, d,
                                                                        c->enc, c->row_in, c->row_out);
    count_launch(), k_scale_weights<float><<<grid_for(md), 256, 0, st>>>(
        (const float*)W_hat, c->rsig, d, md, c->Wt_hi, c->Wt_lo, c->enc, c->row_in, flag);
  } else {
    count_launch(), k_row_scales<__nv_bfloat16><<<grid_for(m, 8), 256, 0, st>>>(
        (const __nv_bfloat16*)W_hat, c->rsig, m, d, c->enc, c->row_in, c->row_out);
    count_launch(), k_scale_weights<__nv_bfloat16><<<grid_for(md), 256, 0, st>>>(
        (const __nv_bfloat16*)W_hat, c->rsig, d, md, c->Wt_hi, c->Wt_lo, c->enc, c->row_in, flag);
  }
  CK(cudaGetLastError());
  c->prepared = true;
  return ADMMQ_OK;
}

int admmq_eigh(admmq_ctx* c, void* stream) {
  if (!c || !c->prepared) return ADMMQ_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int d = c->d;
  int host_status[4] = {0, 0, 0, 0};
  CK(cudaMemcpyAsync(host_status, c->status, 16, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  if (host_status[1] == SETUP_NONFINITE) return ADMMQ_ERR_NONFINITE;
  if (host_status[1] == SETUP_NOT_PD) return ADMMQ_ERR_NOT_PD;
  if (cusolverDnSetStream(c->solver, st) != CUSOLVER_STATUS_SUCCESS) return ADMMQ_ERR_CUDA;
  if (cusolverDnDsyevd(c->solver, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_UPPER, d, c->Ht, d,
                       c->evals, c->work, c->lwork, c->devinfo) != CUSOLVER_STATUS_SUCCESS)
    return ADMMQ_ERR_EIG;
  count_launch(), k_eigvals<<<grid_for(d), 256, 0, st>>>(c->evals, d, c->lam32, c->status);
  CK(cudaGetLastError());
  count_launch(), k_split_eigvecs<<<dim3(cdiv(d, 32), cdiv(d, 32)), dim3(32, 8), 0, st>>>(c->Ht, d, c->E_hi, c->E_lo,
                                                                          c->Q_hi, c->Q_lo, c->enc);
  CK(cudaGetLastError());
  int info = 0;
  CK(cudaMemcpyAsync(&info, c->devinfo, sizeof(int), cudaMemcpyDeviceToHost, st));
  CK(cudaMemcpyAsync(host_status, c->status, 16, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  if (info != 0) return ADMMQ_ERR_EIG;
  if (host_status[2] != 0) return ADMMQ_ERR_NONFINITE;
  c->eig_done = true;
  return ADMMQ_OK;
}

int admmq_setup(admmq_ctx** out, const float* G, const void* W_hat, int w_dtype, int d, int m,
                const admmq_params* p, void* ws, size_t ws_bytes, void* stream) {
  int rc = admmq_create(out, d, m, p, ws, ws_bytes);
  if (rc) return rc;
  rc = admmq_prepare(*out, G, W_hat, w_dtype, stream);
  if (!rc) rc = admmq_eigh(*out, stream);
  if (rc) {
    admmq_destroy(*out);
    *out = nullptr;
  }
  return rc;
}

int admmq_init(admmq_ctx* c, uint8_t* codes, float* scale, float* zero, void* stream) {
  if (!c || !c->eig_done || !codes || !scale || !zero) return ADMMQ_ERR_INVALID_ARG;
  if (!aligned32(codes)) return ADMMQ_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int d = c->d, m = c->m;
  // C0' = Lambda Q^T W^~   (row j, column k)
  GemmGeom g = eig_geom(c->enc, m, d, c->status);
  EpiScaleStore::Params ep{c->C0, c->lam32, c->row_out, d};
  CK((launch_eig<EpiScaleStore, EpiScaleStore, EpiScaleStore>(c->enc, c->mWt, c->mE, g, ep, st)));
  const long long groups = (long long)m * (d / c->p.group);
  int* flag = c->status + 3;
  if (c->w_dtype == ADMMQ_DTYPE_F32)
    count_launch(), k_init_rtn<float><<<grid_for(groups, 8), 256, 0, st>>>(
        (const float*)c->W_hat, c->rsig, m, d, c->p.group, c->L, codes, scale, zero, c->V,
        c->P_hi, c->P_lo, c->enc, c->row_in, flag);
  else
    count_launch(), k_init_rtn<__nv_bfloat16><<<grid_for(groups, 8), 256, 0, st>>>(
        (const __nv_bfloat16*)c->W_hat, c->rsig, m, d, c->p.group, c->L, codes, scale, zero,
        c->V, c->P_hi, c->P_lo, c->enc, c->row_in, flag);
  CK(cudaGetLastError());
  if (c->p.iters > 0) {
    const int T = c->p.iters;
    std::vector<float> tab(2 * (size_t)T);  // rho_t, then the dual factors (adjacent in the workspace)
    for (int t = 0; t < T; ++t) {
      tab[t] = rho_at(c->p, t);
      tab[T + t] = vscale_at(c->p, t);
    }
    CK(cudaMemcpyAsync(c->rho_tab, tab.data(), sizeof(float) * tab.size(), cudaMemcpyHostToDevice, st));
  }
  CK(cudaMemsetAsync(c->ready, 0, sizeof(int) * (2 * cdiv(m, 2 * kBM) + 2), st));
  c->ready_base = 0;
  c->fused_launches = 0;
  c->inited = true;
  return ADMMQ_OK;
}

int admmq_iterate(admmq_ctx* c, int t0, int count, uint8_t* codes, float* scale, float* zero,
                  void* stream) {
  if (!c || !c->inited || !codes || !scale || !zero) return ADMMQ_ERR_INVALID_ARG;
  if (!aligned32(codes)) return ADMMQ_ERR_INVALID_ARG;
  if (t0 < 0 || count < 0 || t0 + count > c->p.iters) return ADMMQ_ERR_INVALID_ARG;
  if (count == 0) return ADMMQ_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const int d = c->d, m = c->m;
  GemmGeom g = eig_geom(c->enc, m, d, c->status);
  int* flag = c->status + 3;
  TUpdateParams p1{c->C0, c->lam32, c->T_hi, c->T_lo, c->row_in, c->row_out, flag, 0.f, d};
  ProjParams p2;
  p2.V = c->V;
  p2.codes = codes;
  p2.scale = scale;
  p2.zero = zero;
  p2.p_hi = c->P_hi;
  p2.p_lo = c->P_lo;
  p2.row_in = c->row_in;
  p2.row_out = c->row_out;
  p2.flag = flag;
  p2.sig = c->sigma;
  p2.rsig = c->rsig;
  p2.hd = c->hdiag;
  p2.part = nullptr;
  p2.wdump = c->wdump;
  p2.ld = d;
  p2.group = c->p.group;
  p2.L = c->L;
  p2.vs = 1.f;
  p2.fit_w = c->p.fit_on_w;
  auto new_event = [&](cudaEvent_t& e) -> int {
    CK(cudaEventCreate(&e));
    return ADMMQ_OK;
  };
  if (c->p.schedule == ADMMQ_SCHEDULE_FUSED) {
    // one launch for all the iterations of the call
    {
      const int t = t0, n = count;
      admmq_ctx::TimingRec rec{nullptr, nullptr, nullptr, true, n};
      if (c->timing) {
        int rc = new_event(rec.a);
        if (!rc) rc = new_event(rec.b);
        if (rc) return rc;
        c->ev.push_back(rec);
        CK(cudaEventRecord(rec.a, st));
      }
      cudaError_t e;
      switch (c->p.grid_mode) {
        case ADMMQ_GRID_MINMAX:
          e = launch_admm_loop_split<GRID_MINMAX>(c, g, p1, p2, t, n, st);
          break;
        case ADMMQ_GRID_LSQ:
          e = launch_admm_loop_split<GRID_LSQ>(c, g, p1, p2, t, n, st);
          break;
        case ADMMQ_GRID_MSE:
          e = launch_admm_loop_split<GRID_MSE>(c, g, p1, p2, t, n, st);
          break;
        default:
          e = launch_admm_loop_split<GRID_FROZEN>(c, g, p1, p2, t, n, st);
          break;
      }
      CK(e);
      c->ready_base += n;
      c->fused_launches += 1;
      if (c->timing) CK(cudaEventRecord(rec.b, st));
    }
    return ADMMQ_OK;
  }
  for (int t = t0; t < t0 + count; ++t) {
    admmq_ctx::TimingRec rec{nullptr, nullptr, nullptr, false, 1};
    if (c->timing) {
      int rc = new_event(rec.a);
      if (!rc) rc = new_event(rec.b);
      if (!rc) rc = new_event(rec.c);
      if (rc) return rc;
      c->ev.push_back(rec);
      CK(cudaEventRecord(rec.a, st));
    }
    p1.rho = rho_at(c->p, t);
    CK((launch_eig<EpiTUpdate<ENC_TF32X3>, EpiTUpdate<ENC_MIX>, EpiTUpdate<ENC_F16>>(c->enc, c->mP,
                                                                                    c->mE, g, p1, st)));
    if (c->timing) CK(cudaEventRecord(rec.b, st));
    p2.part = c->resid_part + (size_t)t * c->tiles_eig * 8;
    p2.vs = vscale_at(c->p, t);
    cudaError_t e;
    switch (c->p.grid_mode) {
      case ADMMQ_GRID_MINMAX:
        e = launch_eig<EpiProject<GRID_MINMAX, ENC_TF32X3>, EpiProject<GRID_MINMAX, ENC_MIX>,
                       EpiProject<GRID_MINMAX, ENC_F16>>(c->enc, c->mT, c->mQ, g, p2, st);
        break;
      case ADMMQ_GRID_LSQ:
        e = launch_eig<EpiProject<GRID_LSQ, ENC_TF32X3>, EpiProject<GRID_LSQ, ENC_MIX>,
                       EpiProject<GRID_LSQ, ENC_F16>>(c->enc, c->mT, c->mQ, g, p2, st);
        break;
      case ADMMQ_GRID_MSE:
        e = launch_eig<EpiProject<GRID_MSE, ENC_TF32X3>, EpiProject<GRID_MSE, ENC_MIX>,
                       EpiProject<GRID_MSE, ENC_F16>>(c->enc, c->mT, c->mQ, g, p2, st);
        break;
      default:
        e = launch_eig<EpiProject<GRID_FROZEN, ENC_TF32X3>, EpiProject<GRID_FROZEN, ENC_MIX>,
                       EpiProject<GRID_FROZEN, ENC_F16>>(c->enc, c->mT, c->mQ, g, p2, st);
        break;
    }
    CK(e);
    if (c->timing) CK(cudaEventRecord(rec.c, st));
  }
  return ADMMQ_OK;
}

int admmq_finish(admmq_ctx* c, const uint8_t* codes, const float* scale, const float* zero,
                 double* resid, double* objective, void* stream) {
  if (!c || !c->inited) return ADMMQ_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int d = c->d, m = c->m;
  if (resid && c->p.iters > 0) {
    count_launch(), k_reduce_resid<<<c->p.iters, 256, 0, st>>>(c->resid_part, c->tiles_eig * 4, (double)c->p.rho0,
                                               (double)c->p.gamma, resid);
    CK(cudaGetLastError());
  }
  if (objective) {
    if (!codes || !scale || !zero) return ADMMQ_ERR_INVALID_ARG;
    const long long md = (long long)m * d;
    int* flag = c->status + 3;
    if (c->w_dtype == ADMMQ_DTYPE_F32)
      count_launch(), k_delta_planes<float><<<grid_for(md), 256, 0, st>>>(
          (const float*)c->W_hat, codes, scale, zero, c->rsig, d, c->p.group, md, c->T_hi, c->T_lo,
          c->enc, c->row_in, flag);
    else
      count_launch(), k_delta_planes<__nv_bfloat16><<<grid_for(md), 256, 0, st>>>(
          (const __nv_bfloat16*)c->W_hat, codes, scale, zero, c->rsig, d, c->p.group, md, c->T_hi,
          c->T_lo, c->enc, c->row_in, flag);
    CK(cudaGetLastError());
    GemmGeom g = eig_geom(c->enc, m, d, c->status);
    EpiObjective::Params ep{c->lam32, c->row_out, c->obj_part};
    CK((launch_eig<EpiObjective, EpiObjective, EpiObjective>(c->enc, c->mT, c->mE, g, ep, st)));
    count_launch(), k_reduce_objective<<<1, 256, 0, st>>>(c->obj_part, c->tiles_eig * 4, objective);
    CK(cudaGetLastError());
  }
  return ADMMQ_OK;
}

int admmq_solve(admmq_ctx* c, uint8_t* codes, float* scale, float* zero, double* resid,
                double* objective, void* stream) {
  int rc = admmq_init(c, codes, scale, zero, stream);
  if (!rc) rc = admmq_iterate(c, 0, c->p.iters, codes, scale, zero, stream);
  if (!rc) rc = admmq_finish(c, codes, scale, zero, resid, objective, stream);
  return rc;
}

int admmq_pack(const uint8_t* codes, int d, int m, int bits, uint32_t* packed, void* stream) {
  if (!codes || !packed || d <= 0 || m <= 0 || d % 32 != 0 || bits < 1 || bits > 8)
    return ADMMQ_ERR_INVALID_ARG;
  if (((uintptr_t)codes & 15) || ((uintptr_t)packed & 15)) return ADMMQ_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const long long groups = (long long)m * (d / 32);
  const int grid = grid_for(groups, 256);  // one group per thread, 8 warps per block
#define PACK_CASE(B)                                                         \
  case B:                                                                    \
    count_launch(), k_pack<B><<<grid, 256, 0, st>>>(codes, groups, packed);  \
    break;
  switch (bits) {
    PACK_CASE(1)
    PACK_CASE(2)
    PACK_CASE(3)
    PACK_CASE(4)
    PACK_CASE(5)
    PACK_CASE(6)
    PACK_CASE(7)
    PACK_CASE(8)
  }
#undef PACK_CASE
  CK(cudaGetLastError());
  return ADMMQ_OK;
}

int admmq_get_buffer(admmq_ctx* c, int which, void** ptr, size_t* bytes) {
  if (!c || !ptr) return ADMMQ_ERR_INVALID_ARG;
  const size_t d = c->d, md = (size_t)c->m * c->d, dd = d * d;
  void* p = nullptr;
  size_t b = 0;
  switch (which) {
    case ADMMQ_BUF_SIGMA: p = c->sigma; b = 4 * d; break;
    case ADMMQ_BUF_RSIG: p = c->rsig; b = 4 * d; break;
    case ADMMQ_BUF_HDIAG: p = c->hdiag; b = 4 * d; break;
    case ADMMQ_BUF_LAMBDA: p = c->lam32; b = 4 * d; break;
    case ADMMQ_BUF_V: p = c->V; b = 4 * md; break;
    case ADMMQ_BUF_C0: p = c->C0; b = 4 * md; break;
    case ADMMQ_BUF_P_HI: p = c->P_hi; b = 4 * md; break;
    case ADMMQ_BUF_P_LO: p = c->P_lo; b = 4 * md; break;
    case ADMMQ_BUF_T_HI: p = c->T_hi; b = 4 * md; break;
    case ADMMQ_BUF_T_LO: p = c->T_lo; b = 4 * md; break;
    case ADMMQ_BUF_E_HI: p = c->E_hi; b = 4 * dd; break;
    case ADMMQ_BUF_E_LO: p = c->E_lo; b = 4 * dd; break;
    case ADMMQ_BUF_HT: p = c->Ht; b = 8 * dd; break;
    case ADMMQ_BUF_STATUS: p = c->status; b = 16; break;
    case ADMMQ_BUF_ROW_IN: p = c->row_in; b = 4 * (size_t)c->m; break;
    case ADMMQ_BUF_ROW_OUT: p = c->row_out; b = 4 * (size_t)c->m; break;
    default: return ADMMQ_ERR_INVALID_ARG;
  }
  *ptr = p;
  if (bytes) *bytes = b;
  return ADMMQ_OK;
}

int admmq_debug_dump_wtilde(admmq_ctx* c, float* wtilde) {
  if (!c || !aligned32(wtilde)) return ADMMQ_ERR_INVALID_ARG;
  c->wdump = wtilde;
  return ADMMQ_OK;
}

int admmq_set_timing(admmq_ctx* c, int enable) {
  if (!c) return ADMMQ_ERR_INVALID_ARG;
  destroy_events(c);
  c->timing = enable != 0;
  return ADMMQ_OK;
}

int admmq_get_timing(admmq_ctx* c, double ms[2], int launches[2], int* iters_timed) {
  if (!c || !ms || !launches) return ADMMQ_ERR_INVALID_ARG;
  ms[0] = ms[1] = 0.0;
  launches[0] = launches[1] = 0;
  int iters = 0;
  for (const auto& r : c->ev) {
    float a = 0.f, b = 0.f;
    CK(cudaEventSynchronize(r.fused ? r.b : r.c));
    CK(cudaEventElapsedTime(&a, r.a, r.b));
    ms[0] += a;
    launches[0] += 1;
    if (!r.fused) {
      CK(cudaEventElapsedTime(&b, r.b, r.c));
      ms[1] += b;
      launches[1] += 1;
    }
    iters += r.iters;
  }
  if (iters_timed) *iters_timed = iters;
  return ADMMQ_OK;
}

int admmq_project(const float* wt, float* V, const float* sig, const float* rsig,
                  const float* hd, int d, int m, int bits, int g, int mode, int split,
                  uint8_t* codes, float* scale, float* zero, void* p_hi, void* p_lo,
                  const float* row_scale, int* range_flag, double* resid, float dual_scale,
                  int fit_on_w, void* stream) {
  if (!wt || !V || !sig || !rsig || !hd || !codes || !scale || !zero || !p_hi || !p_lo || !resid)
    return ADMMQ_ERR_INVALID_ARG;
  if (d <= 0 || m <= 0 || d % 32 != 0 || !(g == 32 || g == 64 || g == 128) || d % g != 0 ||
      bits < 1 || bits > 8 || mode < ADMMQ_GRID_MINMAX || mode > ADMMQ_GRID_MSE ||
      !(split == ADMMQ_SPLIT_3XTF32 || split == ADMMQ_SPLIT_MIXED || split == ADMMQ_SPLIT_F16) ||
      !(dual_scale > 0.f && dual_scale <= 1e30f) || (fit_on_w != 0 && fit_on_w != 1))
    return ADMMQ_ERR_INVALID_ARG;
  if (!aligned32(V) || !aligned32(codes) || !aligned32(p_hi) || !aligned32(p_lo) ||
      ((uintptr_t)wt & 15) || ((uintptr_t)sig & 31) || ((uintptr_t)rsig & 31) || ((uintptr_t)hd & 31) ||
      ((uintptr_t)row_scale & 3) || ((uintptr_t)range_flag & 3))
    return ADMMQ_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  CK(cudaMemsetAsync(resid, 0, 2 * sizeof(double), st));
  const bool staged = mode != ADMMQ_GRID_MSE;
  const int tpg = staged ? g / 32 : 1;
  const int rows = staged ? proj_rows(tpg) : 128;
  const int block = staged ? 32 : 128;
  dim3 grid(cdiv(m, rows), d / g);
  const size_t smem = staged ? sizeof(float) * proj_floats(g, tpg) : 0;  // <= 11,072 bytes
  const int L = (1 << bits) - 1;
  const int enc = split == ADMMQ_SPLIT_MIXED ? ENC_MIX : (split == ADMMQ_SPLIT_F16 ? ENC_F16 : ENC_TF32X3);
#define PROJECT_LAUNCH(MODE, ENC, STAGED, TPG)                                             \
  {                                                                                         \
    int per_sm = 0;                                                                         \
    if (STAGED)                                                                             \
      CK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_project<MODE, ENC, STAGED, TPG>, \
                                                       block, smem));                       \
    /* the L2 prefetch pays for the fp16 split's 4-byte P planes (measured: least  */     \
    /* squares +10%, min/max and frozen +6%); with 8-byte planes it cost 2%         */     \
    const int ahead = (ENC == ENC_F16 && (long long)grid.x * grid.y < (1ll << 31))          \
                          ? num_sms() * per_sm : 0;                                        \
    count_launch(), k_project<MODE, ENC, STAGED, TPG><<<grid, block, smem, st>>>(            \
                        wt, V, sig, rsig, hd, m, d, g, L, codes, scale, zero, p_hi, p_lo,   \
                        row_scale, range_flag, resid, dual_scale, fit_on_w, ahead);         \
  }
#define PROJECT_STAGED(MODE, ENC)      \
  if (tpg == 4) {                      \
    PROJECT_LAUNCH(MODE, ENC, true, 4) \
  } else if (tpg == 2) {               \
    PROJECT_LAUNCH(MODE, ENC, true, 2) \
  } else {                             \
    PROJECT_LAUNCH(MODE, ENC, true, 1) \
  }
#define PROJECT_GLOBAL(MODE, ENC) PROJECT_LAUNCH(MODE, ENC, false, 1)
#define PROJECT_CASE(MODE, KIND) \
  if (enc == ENC_MIX) {          \
    KIND(MODE, ENC_MIX)          \
  } else if (enc == ENC_F16) {   \
    KIND(MODE, ENC_F16)          \
  } else {                       \
    KIND(MODE, ENC_TF32X3)       \
  }
  if (mode == ADMMQ_GRID_MINMAX) {
    PROJECT_CASE(GRID_MINMAX, PROJECT_STAGED)
  } else if (mode == ADMMQ_GRID_LSQ) {
    PROJECT_CASE(GRID_LSQ, PROJECT_STAGED)
  } else if (mode == ADMMQ_GRID_MSE) {
    PROJECT_CASE(GRID_MSE, PROJECT_GLOBAL)
  } else {
    PROJECT_CASE(GRID_FROZEN, PROJECT_STAGED)
  }
#undef PROJECT_CASE
#undef PROJECT_STAGED
#undef PROJECT_GLOBAL
#undef PROJECT_LAUNCH
  CK(cudaGetLastError());
  return ADMMQ_OK;
}

int admmq_split_mode(const admmq_ctx* c) {
  if (!c) return ADMMQ_ERR_INVALID_ARG;
  return c->enc == ENC_MIX ? ADMMQ_SPLIT_MIXED : (c->enc == ENC_F16 ? ADMMQ_SPLIT_F16 : ADMMQ_SPLIT_3XTF32);
}

int admmq_set_split(admmq_ctx* c, int split_mode, void* stream) {
  if (!c || !c->eig_done) return ADMMQ_ERR_INVALID_ARG;
  if (!(split_mode == ADMMQ_SPLIT_3XTF32 || split_mode == ADMMQ_SPLIT_MIXED ||
        split_mode == ADMMQ_SPLIT_F16))
    return ADMMQ_ERR_INVALID_ARG;
  const int enc = split_mode == ADMMQ_SPLIT_MIXED ? ENC_MIX
                  : split_mode == ADMMQ_SPLIT_F16 ? ENC_F16
                                                  : ENC_TF32X3;
  cudaStream_t st = (cudaStream_t)stream;
  const int d = c->d, m = c->m;
  // the operand maps of the new encoding (same buffers: every encoding fits
  // 4 bytes per element per plane)
  CUtensorMap mWt[2], mP[2], mT[2], mE[2], mQ[2];
  bool ok = make_plane_maps(mWt, c->Wt_hi, c->Wt_lo, d, m, kBM, enc) &&
            make_plane_maps(mP, c->P_hi, c->P_lo, d, m, kBM, enc) &&
            make_plane_maps(mT, c->T_hi, c->T_lo, d, m, kBM, enc) &&
            make_plane_maps(mE, c->E_hi, c->E_lo, d, d, EigCfg::B_ROWS, enc) &&
            make_plane_maps(mQ, c->Q_hi, c->Q_lo, d, d, EigCfg::B_ROWS, enc);
  if (!ok) return ADMMQ_ERR_CUDA;
  // clear the timeout and range words; the setup and eigenvalue words stay
  CK(cudaMemsetAsync(c->status, 0, sizeof(int), st));
  CK(cudaMemsetAsync(c->status + 3, 0, sizeof(int), st));
  const long long md = (long long)m * d;
  int* flag = c->status + 3;
  if (c->w_dtype == ADMMQ_DTYPE_F32) {
    count_launch(), k_row_scales<float><<<grid_for(m, 8), 256, 0, st>>>(
        (const float*)c->W_hat, c->rsig, m, d, enc, c->row_in, c->row_out);
    count_launch(), k_scale_weights<float><<<grid_for(md), 256, 0, st>>>(
        (const float*)c->W_hat, c->rsig, d, md, c->Wt_hi, c->Wt_lo, enc, c->row_in, flag);
  } else {
    count_launch(), k_row_scales<__nv_bfloat16><<<grid_for(m, 8), 256, 0, st>>>(
        (const __nv_bfloat16*)c->W_hat, c->rsig, m, d, enc, c->row_in, c->row_out);
    count_launch(), k_scale_weights<__nv_bfloat16><<<grid_for(md), 256, 0, st>>>(
        (const __nv_bfloat16*)c->W_hat, c->rsig, d, md, c->Wt_hi, c->Wt_lo, enc, c->row_in,
        flag);
  }
  CK(cudaGetLastError());
  count_launch(), k_split_eigvecs<<<dim3(cdiv(d, 32), cdiv(d, 32)), dim3(32, 8), 0, st>>>(
      c->Ht, d, c->E_hi, c->E_lo, c->Q_hi, c->Q_lo, enc);
  CK(cudaGetLastError());
  c->enc = enc;
  for (int p = 0; p < 2; ++p) {
    c->mWt[p] = mWt[p];
    c->mP[p] = mP[p];
    c->mT[p] = mT[p];
    c->mE[p] = mE[p];
    c->mQ[p] = mQ[p];
  }
  c->inited = false;  // the iterate's planes are in the old encoding: admmq_init next
  return ADMMQ_OK;
}

int admmq_debug_rint_div(const float* y, const float* s, long long n, float* out, void* stream) {
  if (!y || !s || !out || n < 0 || n % 8 != 0) return ADMMQ_ERR_INVALID_ARG;
  if (n == 0) return ADMMQ_OK;
  cudaStream_t st = (cudaStream_t)stream;
  count_launch(), k_rint_div<<<grid_for(n / 8), 256, 0, st>>>(y, s, n / 8, out);
  CK(cudaGetLastError());
  return ADMMQ_OK;
}

int admmq_debug_skew_ready(admmq_ctx* c, int iterations) {
  if (!c || iterations < 0) return ADMMQ_ERR_INVALID_ARG;
  c->ready_base += iterations;
  return ADMMQ_OK;
}

int admmq_check(admmq_ctx* c, void* stream) {
  if (!c) return ADMMQ_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  int host_status[4] = {0, 0, 0, 0};
  CK(cudaMemcpyAsync(host_status, c->status, 16, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  if (host_status[0] != KSTAT_OK) return ADMMQ_ERR_TIMEOUT;
  if (host_status[3] != 0) return ADMMQ_ERR_RANGE;
  return ADMMQ_OK;
}

// ------------------------------------------------------------------ GPTQ

size_t admmq_gptq_workspace_bytes(int d, int m, int block) {
  if (d <= 0 || m <= 0 || d % 32 != 0 || !(block == 32 || block == 64 || block == 128)) return 0;
  const int lw = gptq_lwork(d);
  if (lw < 0) return 0;
  return gptq_layout(d, m, block, lw).total;
}

int admmq_gptq(const float* G, const void* W_hat, int w_dtype, int d, int m, int bits, int group,
               float lambda_rel, int block, uint8_t* codes, float* scale, float* zero, void* ws,
               size_t ws_bytes, void* stream) {
  if (!G || !W_hat || !codes || !scale || !zero || !ws) return ADMMQ_ERR_INVALID_ARG;
  if (d <= 0 || m <= 0 || d % 32 != 0 || !(group == 32 || group == 64 || group == 128) ||
      d % group != 0 || bits < 1 || bits > 8 || !(lambda_rel >= 0.f) ||
      !(block == 32 || block == 64 || block == 128) ||
      (w_dtype != ADMMQ_DTYPE_F32 && w_dtype != ADMMQ_DTYPE_BF16))
    return ADMMQ_ERR_INVALID_ARG;
  if (((uintptr_t)ws & 255) != 0) return ADMMQ_ERR_INVALID_ARG;
  const int lw = gptq_lwork(d);
  if (lw < 0) return ADMMQ_ERR_CUDA;
  const GptqLayout Lo = gptq_layout(d, m, block, lw);
  if (ws_bytes < Lo.total) return ADMMQ_ERR_WORKSPACE;
  int rc = device_ok();
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* base = (uint8_t*)ws;
  int* status = (int*)(base + Lo.status);
  double* lam64 = (double*)(base + Lo.lam64);
  double* Hd = (double*)(base + Lo.Hd);
  double* Wd = (double*)(base + Lo.Wd);
  double* E = (double*)(base + Lo.E);
  double* work = (double*)(base + Lo.work);
  int* devinfo = (int*)(base + Lo.devinfo);
  const int L = (1 << bits) - 1;

  // H = X^T X + lambda I (lambda as in the ADMM-Q setup) and the fixed grid
  CK(cudaMemsetAsync(status, 0, 16, st));
  count_launch(), k_diag_stats<<<1, 1024, 0, st>>>(G, d, lambda_rel, 1, lam64, (double*)(base + Lo.sig64),
                                                   (float*)(base + Lo.hdiag), (float*)(base + Lo.sigma),
                                                   (float*)(base + Lo.rsig), status);
  CK(cudaGetLastError());
  count_launch(), k_gptq_hessian<<<grid_for((long long)d * d), 256, 0, st>>>(G, d, lam64, Hd);
  CK(cudaGetLastError());
  const long long groups = (long long)m * (d / group);
  if (w_dtype == ADMMQ_DTYPE_F32)
    count_launch(), k_gptq_start<float><<<grid_for(groups, 128), 128, 0, st>>>(
        (const float*)W_hat, m, d, group, L, scale, zero, Wd);
  else
    count_launch(), k_gptq_start<__nv_bfloat16><<<grid_for(groups, 128), 128, 0, st>>>(
        (const __nv_bfloat16*)W_hat, m, d, group, L, scale, zero, Wd);
  CK(cudaGetLastError());
  int host_status[4] = {0, 0, 0, 0};
  CK(cudaMemcpyAsync(host_status, status, 16, cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  if (host_status[1] == SETUP_NONFINITE) return ADMMQ_ERR_NONFINITE;
  if (host_status[1] == SETUP_NOT_PD) return ADMMQ_ERR_NOT_PD;

  // R = upper Cholesky factor of H^-1.  cuSOLVER is column-major: the lower
  // factor it writes is, read row-major, the upper factor R with R^T R = A.
  cusolverDnHandle_t sv = gptq_solver();
  cublasHandle_t bl = gptq_blas();
  if (!sv || !bl) return ADMMQ_ERR_CUDA;
  if (cusolverDnSetStream(sv, st) != CUSOLVER_STATUS_SUCCESS ||
      cublasSetStream(bl, st) != CUBLAS_STATUS_SUCCESS)
    return ADMMQ_ERR_CUDA;
  auto info_ok = [&]() -> int {
    int info = 0;
    if (cudaMemcpyAsync(&info, devinfo, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return ADMMQ_ERR_CUDA;
    return info == 0 ? ADMMQ_OK : ADMMQ_ERR_NOT_PD;
  };
  if (cusolverDnDpotrf(sv, CUBLAS_FILL_MODE_LOWER, d, Hd, d, work, lw, devinfo) !=
      CUSOLVER_STATUS_SUCCESS)
    return ADMMQ_ERR_CUDA;
  if ((rc = info_ok())) return rc;
  if (cusolverDnDpotri(sv, CUBLAS_FILL_MODE_LOWER, d, Hd, d, work, lw, devinfo) !=
      CUSOLVER_STATUS_SUCCESS)
    return ADMMQ_ERR_CUDA;
  if ((rc = info_ok())) return rc;
  if (cusolverDnDpotrf(sv, CUBLAS_FILL_MODE_LOWER, d, Hd, d, work, lw, devinfo) !=
      CUSOLVER_STATUS_SUCCESS)
    return ADMMQ_ERR_CUDA;
  if ((rc = info_ok())) return rc;

  // column blocks: the sequential block kernel, then the trailing update
  //   W[:, b:] -= E R[a:b, b:]   (row-major; column-major C^T = R^T-block E^T)
  const double minus_one = -1.0, one = 1.0;
  for (int a = 0; a < d; a += block) {
    const int bw = d - a < block ? d - a : block;
    count_launch(), k_gptq_block<<<cdiv(m, 8), 256, 0, st>>>(Wd, Hd, scale, zero, m, d, group, L, a,
                                                            bw, codes, E, block);
    CK(cudaGetLastError());
    const int b = a + bw;
    if (b < d) {
      if (cublasDgemm(bl, CUBLAS_OP_N, CUBLAS_OP_N, d - b, m, bw, &minus_one, Hd + (size_t)a * d + b,
                      d, E, block, &one, Wd + b, d) != CUBLAS_STATUS_SUCCESS)
        return ADMMQ_ERR_CUDA;
    }
  }
  CK(cudaGetLastError());
  return ADMMQ_OK;
}

// ------------------------------------------- no-allocation Gram variant

}  // extern "C"

namespace {

// Scratch of admmq_build_hessian_static: a status word (first 256 bytes) and
// the k-split partial sums.  Shared by every call on a device.
__device__ __align__(256) uint8_t g_static_scratch[ADMMQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// The array's device address belongs to the context the module was loaded
// into: after cudaDeviceReset (or any other teardown of the primary context)
// the module is loaded again and the array may sit elsewhere.  So the address
// is cached per device together with the unique id of the context it was
// looked up in, and looked up again whenever the current context differs.
struct StaticSlot {
  unsigned long long ctx_id;  // 0: nothing cached
  void* ptr;
};
StaticSlot g_static_slot[kMaxDevices] = {};
std::mutex g_static_mu;

// Unique id of the calling thread's current context, or 0 when there is none
// (or it was destroyed).  Driver entry points resolved through the runtime,
// so the library needs no link to libcuda.
unsigned long long current_ctx_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static bool resolved = false;
  if (!resolved) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    resolved = true;
  }
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_static_scratch in the current device's current
// context: looked up with cudaGetSymbolAddress on the first call in a
// context (which also creates the primary context if none is current), then
// taken from the cache while that context stays current.
int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ADMMQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ADMMQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mu);
  const unsigned long long id = current_ctx_id();
  StaticSlot& slot = g_static_slot[dev];
  if (id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return ADMMQ_ERR_CUDA;
    const unsigned long long now = current_ctx_id();  // the context the lookup ran in
    slot.ptr = p;
    slot.ctx_id = now;
    *out = p;
    return ADMMQ_OK;
  }
  *out = slot.ptr;
  return ADMMQ_OK;
}

}  // namespace

extern "C" int admmq_build_hessian_static(const void* X, int64_t n, int d, float* H,
                                          int accumulate, void* stream) {
  if ((!X && n > 0) || !H || d <= 0 || d % 32 != 0 || n < 0) return ADMMQ_ERR_INVALID_ARG;
  if (((uintptr_t)X & 15) != 0) return ADMMQ_ERR_INVALID_ARG;
  const size_t dd4 = (size_t)d * d * 4;
  if (256 + dd4 > ADMMQ_STATIC_SCRATCH_BYTES) return ADMMQ_ERR_WORKSPACE;
  int rc = device_ok();
  if (rc) return rc;
  void* base = nullptr;
  rc = static_scratch(&base);
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if (n == 0) {
    if (!accumulate) CK(cudaMemsetAsync(H, 0, dd4, st));
    return ADMMQ_OK;
  }
  int splits = gram_splits(n, d, num_sms());
  while (splits > 1 && 256 + (size_t)splits * dd4 > ADMMQ_STATIC_SCRATCH_BYTES) --splits;
  int* status = (int*)base;
  float* part = (float*)((uint8_t*)base + 256);
  CK(cudaMemsetAsync(status, 0, 16, st));
  CUtensorMap mx;
  if (!make_map(&mx, X, (uint64_t)d, (uint64_t)n, GramCfg::BK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) return ADMMQ_ERR_CUDA;
  GemmGeom g = make_geom(d, d, n, GramCfg::BN, GramCfg::BK, splits, true, status);
  EpiGramPartial::Params ep{part, (long long)d * d, d};
  CK((launch_gemm<GramCfg, EpiGramPartial>(mx, mx, mx, mx, g, ep, st)));
  const int nb = d / 32;
  count_launch(), k_gram_finalize<<<dim3(nb, nb), dim3(32, 8), 0, st>>>(part, splits, (long long)d * d, d, H,
                                                                          accumulate, status);
  CK(cudaGetLastError());
  return ADMMQ_OK;
}
