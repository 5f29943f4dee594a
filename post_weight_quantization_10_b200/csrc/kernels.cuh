// kernels.cuh -- element-wise, reduction and epilogue kernels of the ADMM-Q
// layer solve (everything that is not the tcgen05 main loop).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "gemm.cuh"

namespace admmq {

enum { GRID_MINMAX = 0, GRID_LSQ = 1, GRID_FROZEN = 2, GRID_MSE = 3 };

// Clipping search of the MSE grid refresh: ratios (32 - k) / 32, k < 16.
constexpr int kClipCandidates = 16;

// ------------------------------------------------------------ small helpers

__device__ __forceinline__ uint16_t bf16_bits(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
// Round a float32 to tf32 (10 explicit mantissa bits), nearest-even, kept in
// a float32 word with the 13 low bits zero.
__device__ __forceinline__ float tf32_rne(float x) {
  uint32_t b = __float_as_uint(x);
  b = (b + 0xFFFu + ((b >> 13) & 1u)) & ~0x1FFFu;
  return __uint_as_float(b);
}
// Operand encodings of the eigenbasis GEMMs (ENC_*, selected by the split
// precision):
//   ENC_TF32X3 (GemmCfg KIND_TF32): plane 0 hi = tf32(x) in fp32 words,
//     plane 1 lo = tf32(x - hi), both fp32 [rows][K];
//   ENC_MIX (KIND_MIX): plane 0 hi = tf32(x) fp32 [rows][K]; plane 1 bf16(hi)
//     and bf16(lo), lo = x - hi (exact in float32), in correction rows of 64
//     bf16 per 32 columns, [rows][2K]: A operands [hi x32 | lo x32], B
//     operands [lo x32 | hi x32];
//   ENC_F16 (KIND_F16X3): plane 0 hi = fp16(x s), plane 1 lo = fp16(x s - hi),
//     both u16 [rows][K], with a power-of-two scale s: 2^14 for B operands
//     (eigenvector entries, |x| <= 1) and the row's own scale for A operands
//     (see k_row_scales); a scaled value at or beyond fp16's largest finite
//     value raises the range flag instead of passing as infinity.
enum { ENC_TF32X3 = 0, ENC_MIX = 1, ENC_F16 = 2 };
constexpr int kBScaleExp = 14;       // B operands of the fp16 split are scaled by 2^14
constexpr float kF16Limit = 65504.f;  // largest finite fp16

// x ~= hi + lo: hi = tf32(x), lo = tf32(x - hi)  (the 3xTF32 planes).
__device__ __forceinline__ void split2(float x, float& hi, float& lo) {
  hi = tf32_rne(x);
  lo = tf32_rne(__fsub_rn(x, hi));
}
__device__ __forceinline__ void split_mix(float x, float& hi, uint16_t& hb, uint16_t& lb) {
  hi = tf32_rne(x);
  hb = bf16_bits(hi);
  lb = bf16_bits(__fsub_rn(x, hi));
}
// fp16 pair of an already scaled value: hi = fp16(xs), lo = fp16(xs - hi)
// (xs - hi is exact in float32); both round to nearest even.
__device__ __forceinline__ void split_f16(float xs, uint16_t& hb, uint16_t& lb) {
  const __half h = __float2half_rn(xs);
  hb = __half_as_ushort(h);
  lb = __half_as_ushort(__float2half_rn(__fsub_rn(xs, __half2float(h))));
}
__device__ __forceinline__ uint32_t half2_bits(__half2 h) {
  return (uint32_t)__half_as_ushort(__low2half(h)) |
         ((uint32_t)__half_as_ushort(__high2half(h)) << 16);
}
// Index of column c's hi entry in its correction row (lo is 32 further on
// for A operands, 32 before for B operands).
__device__ __forceinline__ long long cplane_hi(long long c, bool b_side) {
  return 64 * (c >> 5) + (c & 31) + (b_side ? 32 : 0);
}
// Eight consecutive 16-bit words (16 bytes, 16-byte aligned).
__device__ __forceinline__ void st_u16x8(uint16_t* p, const uint16_t (&v)[8]) {
  uint4 u;
  u.x = (uint32_t)v[0] | ((uint32_t)v[1] << 16);
  u.y = (uint32_t)v[2] | ((uint32_t)v[3] << 16);
  u.z = (uint32_t)v[4] | ((uint32_t)v[5] << 16);
  u.w = (uint32_t)v[6] | ((uint32_t)v[7] << 16);
  *reinterpret_cast<uint4*>(p) = u;
}
// Start of row `row` (K = ld columns) in plane 0 / plane 1 of an encoding.
__device__ __forceinline__ void* plane0_row(int enc, void* p0, long long row, int ld) {
  return enc == ENC_F16 ? (void*)(reinterpret_cast<uint16_t*>(p0) + row * ld)
                        : (void*)(reinterpret_cast<float*>(p0) + row * ld);
}
__device__ __forceinline__ void* plane1_row(int enc, void* p1, long long row, int ld) {
  return enc == ENC_TF32X3 ? (void*)(reinterpret_cast<float*>(p1) + row * ld)
                           : (void*)(reinterpret_cast<uint16_t*>(p1) + row * (enc == ENC_MIX ? 2 : 1) * ld);
}
// The same for column c (c % 32 == 0 for the mixed correction rows).
__device__ __forceinline__ void* plane0_at(int enc, void* p0, long long row, int ld, long long c) {
  return enc == ENC_F16 ? (void*)(reinterpret_cast<uint16_t*>(p0) + row * ld + c)
                        : (void*)(reinterpret_cast<float*>(p0) + row * ld + c);
}
__device__ __forceinline__ void* plane1_at(int enc, void* p1, long long row, int ld, long long c) {
  if (enc == ENC_TF32X3) return reinterpret_cast<float*>(p1) + row * ld + c;
  if (enc == ENC_MIX) return reinterpret_cast<uint16_t*>(p1) + row * 2 * ld + 2 * c;
  return reinterpret_cast<uint16_t*>(p1) + row * ld + c;
}
// Columns c..c+7 (c % 8 == 0) of one A-side operand row in the encoding:
// hi_row / lo_row point at the row's (or the column block's) start in planes
// 0 / 1; s is the row's scale (fp16 split only), flag the range flag.
template <int ENC>
__device__ __forceinline__ void put_operand8(void* hi_row, void* lo_row, long long c,
                                             const float (&x)[8], float s, int* flag) {
  if (ENC == ENC_F16) {
    // two elements per conversion: cvt.rn.f16x2.f32 rounds each one to
    // nearest even, as split_f16 does, and leaves them packed (element 2j
    // in the low half, the layout of the plane)
    uint32_t hw[4], lw[4];
    bool bad = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __fmul_rn(x[2 * j], s), b = __fmul_rn(x[2 * j + 1], s);
      bad |= !(fabsf(a) < kF16Limit);
      bad |= !(fabsf(b) < kF16Limit);
      const __half2 h = __floats2half2_rn(a, b);
      const float2 hf = __half22float2(h);
      const __half2 l = __floats2half2_rn(__fsub_rn(a, hf.x), __fsub_rn(b, hf.y));
      hw[j] = half2_bits(h);
      lw[j] = half2_bits(l);
    }
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(hi_row) + c) =
        make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(lo_row) + c) =
        make_uint4(lw[0], lw[1], lw[2], lw[3]);
    if (bad && flag) *flag = 1;
    return;
  }
  float hi[8];
  if (ENC == ENC_MIX) {
    uint16_t hb[8], lb[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) split_mix(x[k], hi[k], hb[k], lb[k]);
    uint16_t* cr = reinterpret_cast<uint16_t*>(lo_row) + cplane_hi(c, false);
    st_u16x8(cr, hb);
    st_u16x8(cr + 32, lb);
  } else {
    float lo[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) split2(x[k], hi[k], lo[k]);
    st_v8f(reinterpret_cast<float*>(lo_row) + c, lo);
  }
  st_v8f(reinterpret_cast<float*>(hi_row) + c, hi);
}
// One A-side element (column c of a row) for element-wise kernels.
__device__ __forceinline__ void put_a1(int enc, void* hi_row, void* lo_row, long long c, float x,
                                       float s, int* flag) {
  if (enc == ENC_F16) {
    const float xs = __fmul_rn(x, s);
    if (!(fabsf(xs) < kF16Limit) && flag) *flag = 1;
    uint16_t hb, lb;
    split_f16(xs, hb, lb);
    reinterpret_cast<uint16_t*>(hi_row)[c] = hb;
    reinterpret_cast<uint16_t*>(lo_row)[c] = lb;
    return;
  }
  const float h = tf32_rne(x), lo = __fsub_rn(x, h);
  reinterpret_cast<float*>(hi_row)[c] = h;
  if (enc == ENC_MIX) {
    uint16_t* cr = reinterpret_cast<uint16_t*>(lo_row) + cplane_hi(c, false);
    cr[0] = bf16_bits(h);
    cr[32] = bf16_bits(lo);
  } else {
    reinterpret_cast<float*>(lo_row)[c] = tf32_rne(lo);
  }
}
// One B-side element from a float64 value (eigenvectors): the low part is
// taken from the float64 residual.
__device__ __forceinline__ void put_b1(int enc, void* hi_row, void* lo_row, long long c, double e) {
  if (enc == ENC_F16) {
    const double xs = e * (double)(1 << kBScaleExp);
    const __half h = __double2half(xs);
    reinterpret_cast<uint16_t*>(hi_row)[c] = __half_as_ushort(h);
    reinterpret_cast<uint16_t*>(lo_row)[c] =
        __half_as_ushort(__double2half(xs - (double)__half2float(h)));
    return;
  }
  const float h = tf32_rne((float)e), lo = (float)(e - (double)h);
  reinterpret_cast<float*>(hi_row)[c] = h;
  if (enc == ENC_MIX) {
    uint16_t* cr = reinterpret_cast<uint16_t*>(lo_row) + cplane_hi(c, true);
    cr[0] = bf16_bits(h);
    cr[-32] = bf16_bits(lo);
  } else {
    reinterpret_cast<float*>(lo_row)[c] = tf32_rne(lo);
  }
}
// clamp to [0, L]; adding +0 turns a -0 into +0 so the result never depends
// on which zero fmaxf returns for (-0, +0)
__device__ __forceinline__ float clampq(float q, float L) {
  return __fadd_rn(fminf(fmaxf(q, 0.f), L), 0.f);
}

// rint(y / s) for eight values sharing the divisor s, with the quotient
// correctly rounded first (the same integers as rintf(__fdiv_rn(y, s))), from
// r = __frcp_rn(s).  t = y r differs from the rounded quotient by at most
// 1.5 * 2^-23 |y / s| (the reciprocal's and the product's roundings, 2^-24
// each, and the quotient's own), so when |t - rint(t)| is below the
// threshold 0.5 - 2^-21 |t| (one fused multiply-add, rounded once) both
// round to the same integer.  Otherwise (a near-tie, a negative threshold
// for |t| >= 2^20, or a non-finite t) that value is divided exactly.  The
// eight fast paths are straight-line code; the exact divisions are rare.
__device__ __forceinline__ bool rint_fast_ok(float t, float q) {
  return fabsf(__fsub_rn(t, q)) < __fmaf_rn(-4.76837158203125e-7f, fabsf(t), 0.5f);  // 2^-21
}
// The rare exact path, out of line: inlined, its eight divisions per batch
// would sit between the hot instructions and spread them in the
// instruction cache.
__device__ __noinline__ float rint_div_exact(float y, float s) { return rintf(__fdiv_rn(y, s)); }
__device__ __forceinline__ void rint_div8(const float (&y)[8], float s, float r, float (&q)[8]) {
  bool exact = false;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float t = __fmul_rn(y[k], r);
    q[k] = rintf(t);
    exact |= !rint_fast_ok(t, q[k]);
  }
  if (exact) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float t = __fmul_rn(y[k], r);
      if (!rint_fast_ok(t, rintf(t))) q[k] = rint_div_exact(y[k], s);
    }
  }
}

// Codes as bytes without float-to-integer conversions: for an integer q in
// [0, 255], q + 2^23 is exact and its low byte is q; for a byte b, the word
// 0x4B0000bb is 2^23 + b.
__device__ __forceinline__ uint32_t code_word(float q) { return __float_as_uint(__fadd_rn(q, 8388608.f)); }
__device__ __forceinline__ uint32_t pack_codes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}
__device__ __forceinline__ float code_at(uint32_t w, int k) {  // byte k (0..3) of w
  return __fsub_rn(__uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u + (uint32_t)k)), 8388608.f);
}

// eight consecutive read-only floats (per-column vectors: sigma, 1/sigma, diag H)
__device__ __forceinline__ void load8_ro(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Eight floats of a per-column vector (sigma, 1/sigma, diag(H)): through the
// read-only path from global memory, or from a copy in shared memory.
template <bool SMEM>
__device__ __forceinline__ void load8_col(const float* p, float (&v)[8]) {
  if (SMEM) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    load8_ro(p, v);
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------- grid fit + projection (fp32)
//
// The D-update's float32 arithmetic, one thread per (row, group).  Every
// operation is an explicitly rounded IEEE op (no contraction) so that the
// result is reproducible bit for bit by a float32 reference:
//   t = W~ + V~,  y = sigma t
//   minmax: mn = min(0, min y), mx = max(0, max y), s = (mx - mn)/L,
//           z = rint(-mn/s)   (s = 1, z = 0 when mx = mn)
//   lsq:    q0 = clamp(rint(y/s_prev) + z_prev); weighted sums (w = diag H)
//           per 32-column block in element order, block sums added
//           pairwise; slope/offset, integer zero point, slope again
//   q = clamp(rint(y/s) + z, 0, L);  D = s (q - z);  D~ = D rsig
//   V~' = t - D~;  P = D~ - V~'  (stored in the GEMM operand encoding)

struct ProjRow {
  float* V;            // this row's V~ at the group's first column
  const float* sig;    // sigma, rsig, diag(H) at the group's first column
  const float* rsig;
  const float* hd;
  uint8_t* codes;
  void* phi;           // P plane 0 at the group's first column (any encoding)
  void* plo;           // P plane 1 at the group's first column
  float* scale;        // this group's scale / zero
  float* zero;
  // COLS_SMEM: copies of the previous codes (the row's, at the group's first
  // column) and of the group's scale and zero point in shared memory
  const uint8_t* codes_in;
  const float* scale_in;
  const float* zero_in;
  float* wdump;        // optional raw W~ output
  float rs;            // the row's operand scale (fp16 split; 1 otherwise)
  float vs;            // dual rescaling rho_t / rho_{t+1} (1 without it)
  int fit_w;           // 1: refresh the grid from sigma W~ (V~ left out of the fit)
  int* flag;           // range flag of the fp16 split
  bool valid;
  bool grid_out;       // this thread stores the group's scale and zero point
};

// Grid spanning [mn, mx] (mn <= 0 <= mx): s = (mx - mn) / L, z = rint(-mn / s);
// an empty range gets s = 1, z = 0.
__device__ __forceinline__ void range_grid(float mn, float mx, float Lf, float& s, float& z) {
  s = __fdiv_rn(__fsub_rn(mx, mn), Lf);
  if (s == 0.f) {
    s = 1.f;
    z = 0.f;
  } else {
    z = __fadd_rn(rintf(__fdiv_rn(-mn, s)), 0.f);
  }
}

// MSE clipping search over one group: candidate k is the grid of the clipped
// range (a mn, a mx), a = (32 - k) / 32; its error sum (y - D)^2 is accumulated
// in element order with every product and sum rounded on its own; the first
// smallest error wins.  The group is read once per 32-column chunk; the
// candidates run in an outer loop over the chunk's y held in registers.
template <bool COLS_SMEM, class LoadW, class LoadV>
__device__ __forceinline__ void mse_clip_grid(LoadW& loadw, LoadV& loadv, const ProjRow& r, int g,
                                              float Lf, float mn, float mx, float& s, float& z) {
  float ce[kClipCandidates];
#pragma unroll
  for (int k = 0; k < kClipCandidates; ++k) ce[k] = 0.f;
#pragma unroll 1
  for (int c = 0; c < g; c += 32) {
    float y[32];
    loadw(c, y);
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
      float vv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (!r.fit_w) loadv(c + e, vv);  // the grid fitted on sigma W~ alone (fit_w)
      float ss[8];
      load8_col<COLS_SMEM>(r.sig + c + e, ss);
#pragma unroll
      for (int j = 0; j < 8; ++j) y[e + j] = __fmul_rn(ss[j], __fadd_rn(y[e + j], vv[j]));
    }
#pragma unroll 1
    for (int k = 0; k < kClipCandidates; ++k) {
      const float a = __fmul_rn((float)(32 - k), 0.03125f);
      float sk, zk;
      range_grid(__fmul_rn(a, mn), __fmul_rn(a, mx), Lf, sk, zk);
      float ek = ce[k];
      const float rk = __frcp_rn(sk);
#pragma unroll
      for (int j0 = 0; j0 < 32; j0 += 8) {
        float y8[8], q8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) y8[j] = y[j0 + j];
        rint_div8(y8, sk, rk, q8);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float q = clampq(__fadd_rn(q8[j], zk), Lf);
          const float dd = __fsub_rn(y8[j], __fmul_rn(sk, __fsub_rn(q, zk)));
          ek = __fadd_rn(ek, __fmul_rn(dd, dd));
        }
      }
      ce[k] = ek;
    }
  }
  float best = ce[0];
  range_grid(mn, mx, Lf, s, z);
#pragma unroll 1
  for (int k = 1; k < kClipCandidates; ++k) {
    if (ce[k] < best) {
      best = ce[k];
      const float a = __fmul_rn((float)(32 - k), 0.03125f);
      range_grid(__fmul_rn(a, mn), __fmul_rn(a, mx), Lf, s, z);
    }
  }
}

// loadw(c, w[32]) gives W~ at columns c .. c + 31 of the group, loadv(c,
// v[8]) the dual V~ at c .. c + 7 (left at zero for an invalid row); the new
// V~ is stored through r.V.  COLS_SMEM: r.sig, r.rsig and r.hd point into
// shared memory.
//
// The least-squares sums are taken over consecutive 32-column blocks, each in
// element order, and the block sums are then added pairwise: (B0 + B1) +
// (B2 + B3) for g = 128, B0 + B1 for 64, B0 for 32.  TPG > 1: that many lanes
// share the group (TPG = g / 32), one block each (columns 0 .. 31 of r's
// pointers, which the caller offsets to the block), lanes rr + (32 / TPG) j
// for block j; the block sums (and min/max) are combined by shuffles in the
// same pairwise order, every lane fits the same grid, and the lane with
// r.grid_out stores it.  Every lane of the warp must call it then.
template <int MODE, int ENC, bool COLS_SMEM = false, int TPG = 1, class LoadW, class LoadV>
__device__ __forceinline__ void project_group(LoadW&& loadw, LoadV&& loadv, const ProjRow& r,
                                              int g, int L, float& r2, float& s2) {
  static_assert(TPG == 1 || MODE != GRID_MSE, "the clipping search keeps one thread per group");
  static_assert(TPG == 1 || TPG == 2 || TPG == 4, "one to four 32-column blocks per group");
  const float Lf = (float)L;
  const int n = TPG > 1 ? 32 : g;  // columns of this thread
  float s0 = 1.f, z0 = 0.f;
  if (r.valid) {  // L2 reads: another SM may have written them in this launch
    s0 = COLS_SMEM ? *r.scale_in : __ldcg(r.scale);
    z0 = COLS_SMEM ? *r.zero_in : __ldcg(r.zero);
  }
  float s = s0, z = z0;
  const float r0 = __frcp_rn(s0);
  if (MODE != GRID_FROZEN) {
    float mn = 0.f, mx = 0.f;
    float Sw = 0.f, Sq = 0.f, Sqq = 0.f, Sy = 0.f, Sqy = 0.f;
    // one thread per group: the last even block (E) and the first pair (A)
    float Ew = 0.f, Eq = 0.f, Eqq = 0.f, Ey = 0.f, Eqy = 0.f;
    float Aw = 0.f, Aq = 0.f, Aqq = 0.f, Ay = 0.f, Aqy = 0.f;
#pragma unroll
    for (int c = 0; c < n; c += 32) {
      float w[32];
      loadw(c, w);
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        float vv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (!r.fit_w) loadv(c + e, vv);  // the grid fitted on sigma W~ alone (fit_w)
        float ss[8], hh[8], y8[8], q8[8];
        load8_col<COLS_SMEM>(r.sig + c + e, ss);
        if (MODE == GRID_LSQ) load8_col<COLS_SMEM>(r.hd + c + e, hh);
#pragma unroll
        for (int k = 0; k < 8; ++k) y8[k] = __fmul_rn(ss[k], __fadd_rn(w[e + k], vv[k]));
        if (MODE == GRID_LSQ) rint_div8(y8, s0, r0, q8);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float y = y8[k];
          if (MODE == GRID_MINMAX || MODE == GRID_MSE) {
            mn = fminf(mn, y);
            mx = fmaxf(mx, y);
          } else {
            const float q0 = clampq(__fadd_rn(q8[k], z0), Lf);
            const float wi = hh[k];
            const float wq = __fmul_rn(wi, q0);
            Sw = __fadd_rn(Sw, wi);
            Sq = __fadd_rn(Sq, wq);
            Sqq = __fadd_rn(Sqq, __fmul_rn(wq, q0));
            Sy = __fadd_rn(Sy, __fmul_rn(wi, y));
            Sqy = __fadd_rn(Sqy, __fmul_rn(wq, y));
          }
        }
      }
      if (MODE == GRID_LSQ && TPG == 1) {  // block c / 32 ends: pairwise combination
        if (c & 32) {  // odd block: its pair is E + S
          Sw = __fadd_rn(Ew, Sw); Sq = __fadd_rn(Eq, Sq); Sqq = __fadd_rn(Eqq, Sqq);
          Sy = __fadd_rn(Ey, Sy); Sqy = __fadd_rn(Eqy, Sqy);
          if (c & 64) {  // the second pair: the total of four blocks stays in S
            Sw = __fadd_rn(Aw, Sw); Sq = __fadd_rn(Aq, Sq); Sqq = __fadd_rn(Aqq, Sqq);
            Sy = __fadd_rn(Ay, Sy); Sqy = __fadd_rn(Aqy, Sqy);
          } else {
            Aw = Sw; Aq = Sq; Aqq = Sqq; Ay = Sy; Aqy = Sqy;
            Sw = 0.f; Sq = 0.f; Sqq = 0.f; Sy = 0.f; Sqy = 0.f;
          }
        } else {
          Ew = Sw; Eq = Sq; Eqq = Sqq; Ey = Sy; Eqy = Sqy;
          Sw = 0.f; Sq = 0.f; Sqq = 0.f; Sy = 0.f; Sqy = 0.f;
        }
      }
    }
    if (MODE == GRID_LSQ) {
      if (TPG == 1) {
        if (g == 32) {
          Sw = Ew; Sq = Eq; Sqq = Eqq; Sy = Ey; Sqy = Eqy;
        } else if (g == 64) {
          Sw = Aw; Sq = Aq; Sqq = Aqq; Sy = Ay; Sqy = Aqy;
        }
      } else {  // lanes 32/TPG apart hold adjacent blocks; the sums are commutative
#pragma unroll
        for (int o = 32 / TPG; o < 32; o <<= 1) {
          Sw = __fadd_rn(Sw, __shfl_xor_sync(0xffffffffu, Sw, o));
          Sq = __fadd_rn(Sq, __shfl_xor_sync(0xffffffffu, Sq, o));
          Sqq = __fadd_rn(Sqq, __shfl_xor_sync(0xffffffffu, Sqq, o));
          Sy = __fadd_rn(Sy, __shfl_xor_sync(0xffffffffu, Sy, o));
          Sqy = __fadd_rn(Sqy, __shfl_xor_sync(0xffffffffu, Sqy, o));
        }
      }
    } else if (TPG > 1 && MODE == GRID_MINMAX) {
#pragma unroll
      for (int o = 32 / TPG; o < 32; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
    }
    if constexpr (MODE == GRID_MINMAX) {
      range_grid(mn, mx, Lf, s, z);
    } else if constexpr (MODE == GRID_MSE) {
      mse_clip_grid<COLS_SMEM>(loadw, loadv, r, g, Lf, mn, mx, s, z);
    } else {
      const float qm = __fdiv_rn(Sq, Sw);
      const float ym = __fdiv_rn(Sy, Sw);
      const float var = __fsub_rn(Sqq, __fmul_rn(Sq, qm));
      const float cov = __fsub_rn(Sqy, __fmul_rn(Sq, ym));
      if (var > 0.f && cov > 0.f) {
        const float s1 = __fdiv_rn(cov, var);
        const float zc = clampq(rintf(__fsub_rn(qm, __fdiv_rn(ym, s1))), Lf);
        const float num = __fsub_rn(Sqy, __fmul_rn(zc, Sy));
        const float den = __fadd_rn(__fsub_rn(Sqq, __fmul_rn(__fmul_rn(2.f, zc), Sq)),
                                    __fmul_rn(__fmul_rn(zc, zc), Sw));
        s = (den > 0.f && num > 0.f) ? __fdiv_rn(num, den) : s1;
        z = zc;
      }
    }
  }
  const float rs = __frcp_rn(s);
#pragma unroll
  for (int c = 0; c < n; c += 32) {
    float w[32];
    loadw(c, w);
    uint32_t cw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // the 32 previous codes
    if (r.valid) {
      if (COLS_SMEM) {
        const uint4 a = *reinterpret_cast<const uint4*>(r.codes_in + c);
        const uint4 b = *reinterpret_cast<const uint4*>(r.codes_in + c + 16);
        cw[0] = a.x; cw[1] = a.y; cw[2] = a.z; cw[3] = a.w;
        cw[4] = b.x; cw[5] = b.y; cw[6] = b.z; cw[7] = b.w;
      } else {
        ld_v8(r.codes + c, cw);
      }
    }
    uint32_t qw[8];
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
      float vv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      loadv(c + e, vv);
      float ss[8], rr[8], t8[8], y8[8], q8[8];
      load8_col<COLS_SMEM>(r.sig + c + e, ss);
      load8_col<COLS_SMEM>(r.rsig + c + e, rr);
      float vn[8], pv[8];
      uint32_t qb[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        t8[k] = __fadd_rn(w[e + k], vv[k]);
        y8[k] = __fmul_rn(ss[k], t8[k]);
      }
      rint_div8(y8, s, rs, q8);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float t = t8[k];
        const float q = clampq(__fadd_rn(q8[k], z), Lf);
        const float D = __fmul_rn(s, __fsub_rn(q, z));
        const float dt = __fmul_rn(D, rr[k]);
        vn[k] = __fmul_rn(__fsub_rn(t, dt), r.vs);
        pv[k] = __fsub_rn(dt, vn[k]);
        qb[k] = code_word(q);
        const float e1 = w[e + k] - dt;
        r2 += e1 * e1;
        // the previous iterate D~_prev = s0 (q_prev - z0) rsig, for the residual
        const float qp = code_at(cw[(e + k) >> 2], (e + k) & 3);
        const float dtp = __fmul_rn(__fmul_rn(s0, __fsub_rn(qp, z0)), rr[k]);
        const float e2 = dt - dtp;
        s2 += e2 * e2;
      }
      qw[e / 4] = pack_codes4(qb[0], qb[1], qb[2], qb[3]);
      qw[e / 4 + 1] = pack_codes4(qb[4], qb[5], qb[6], qb[7]);
      if (r.valid) {
        st_v8f(r.V + c + e, vn);
        put_operand8<ENC>(r.phi, r.plo, c + e, pv, r.rs, r.flag);  // P, A side
        if (r.wdump) {
          float wd[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) wd[k] = w[e + k];
          st_v8f(r.wdump + c + e, wd);
        }
      }
    }
    if (r.valid) st_v8(r.codes + c, qw);
  }
  if (r.valid && r.grid_out) {
    *r.scale = s;
    *r.zero = z;
  }
  if (!r.valid) {  // rows past d_out contribute nothing
    r2 = 0.f;
    s2 = 0.f;
  }
}

// -------------------------------------------------------------- epilogues
// Each epilogue thread owns one accumulator row (tile row rit = 32 q + lane
// of 128-row tile tm) and 128 consecutive columns col0 .. col0 + 127: from
// registers (apply_regs) or from tensor memory (apply_tmem, 32 columns per
// load).

// Gram: raw fp32 tile into the k-split's partial buffer (upper part used).
struct EpiGramPartial {
  static constexpr bool FROM_TMEM = false;
  struct Params {
    float* part;
    long long split_stride;  // elements between k-split buffers
    int ld;
  };
  // From registers: 128 columns starting at col0 of tile row `rit`.
  __device__ static void apply_regs(const Params& p, const GemmGeom& g, const float (&acc)[128],
                                    int tm, int, int split, int rit, int col0) {
    const int row = tm * 128 + rit;
    if (row >= g.M) return;
    float* out = p.part + split * p.split_stride + (long long)row * p.ld;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = col0 + 32 * j;
      if (col < g.N) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<float4*>(out + col + 4 * k) =
              make_float4(acc[32 * j + 4 * k], acc[32 * j + 4 * k + 1], acc[32 * j + 4 * k + 2],
                          acc[32 * j + 4 * k + 3]);
      }
    }
  }
};

// C0' = Lambda (Q^T W^~): column k scaled by lambda_k, stored fp32.
struct EpiScaleStore {
  static constexpr bool FROM_TMEM = false;
  struct Params {
    float* out;
    const float* lam;
    const float* row_out;  // per-row factor that unscales the GEMM result
    int ld;
  };
  // From registers: 128 columns of tile row `rit`, starting at column col0.
  __device__ static void apply_regs(const Params& p, const GemmGeom& g, const float (&acc)[128],
                                    int tm, int, int, int rit, int col0) {
    const int row = tm * 128 + rit;
    if (row >= g.M) return;
    float* o = p.out + (long long)row * p.ld;
    const float ro = p.row_out[row];
#pragma unroll
    for (int c = 0; c < 128; c += 8) {
      const int col = col0 + c;
      if (col < g.N) {
        float l[8], v[8];
        load8_ro(p.lam + col, l);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = __fmul_rn(l[k], __fmul_rn(acc[c + k], ro));
        st_v8f(o + col, v);
      }
    }
  }
};

// GEMM 1 epilogue: T = (C0' + rho acc) / (lambda + rho), stored in the
// operand encoding (A side).
struct TUpdateParams {
  const float* c0;
  const float* lam;
  void* t_hi;             // plane 0 (encoding per the epilogue's ENC)
  void* t_lo;             // plane 1
  const float* row_in;    // per-row operand scale of the fp16 split (1 otherwise)
  const float* row_out;   // per-row factor that unscales a GEMM result row
  int* flag;              // range flag of the fp16 split
  float rho;
  int ld;
};

template <int ENC>
struct EpiTUpdate {
  static constexpr bool FROM_TMEM = false;
  using Params = TUpdateParams;
  __device__ static void apply_regs(const Params& p, const GemmGeom& g, const float (&acc)[128],
                                    int tm, int, int, int rit, int col0) {
    const int row = tm * 128 + rit;
    if (row >= g.M) return;
    const long long rb = (long long)row * p.ld;
    void* hi = plane0_row(ENC, p.t_hi, row, p.ld);
    void* lo = plane1_row(ENC, p.t_lo, row, p.ld);
    const float ro = p.row_out[row], ri = p.row_in[row];
#pragma unroll
    for (int c = 0; c < 128; c += 8) {
      const int col = col0 + c;
      if (col < g.N) {
        float cc[8], ll[8], tv[8];
        ld_v8f(p.c0 + rb + col, cc);
        load8_ro(p.lam + col, ll);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float inv = __frcp_rn(__fadd_rn(ll[j], p.rho));
          const float a = __fmul_rn(acc[c + j], ro);
          tv[j] = __fmul_rn(__fadd_rn(cc[j], __fmul_rn(p.rho, a)), inv);
        }
        put_operand8<ENC>(hi, lo, col, tv, ri, p.flag);
      }
    }
  }
};

// GEMM 2 epilogue: W~ = Q T from tensor memory, fused grid refresh,
// projection, dual update and residual partial sums (one per tile and warp).
struct ProjParams {
  float* V;
  uint8_t* codes;
  float* scale;
  float* zero;
  void* p_hi;     // plane 0 (encoding per the epilogue's ENC)
  void* p_lo;     // plane 1
  const float* row_in;    // per-row operand scale of the fp16 split (1 otherwise)
  const float* row_out;   // per-row factor that unscales W~ = Q T
  int* flag;              // range flag of the fp16 split
  const float* sig;
  const float* rsig;
  const float* hd;
  float* part;    // [tiles][4][2] for this iteration
  float* wdump;   // optional
  float vs;       // dual rescaling of this iteration (1 without it)
  int fit_w;      // grid refreshed from sigma W~ instead of sigma (W~ + V~)
  int ld;         // d_in
  int group;
  int L;
};

template <int MODE, int ENC>
struct EpiProject {
  // The projection keeps a whole group of one row in flight twice (refit and
  // projection passes): it reads the tile from tensor memory, where the
  // engine leaves the summed accumulator, instead of 128 live registers.
  static constexpr bool FROM_TMEM = true;
  using Params = ProjParams;
  // Tile row `rit` of 128-row tile tm, columns col0 .. col0 + 127 at taddr.
  __device__ static void apply_tmem(const Params& p, const GemmGeom& g, uint32_t taddr, int tm,
                                    int rit, int col0) {
    const int row = tm * 128 + rit;
    const bool valid = row < g.M;
    const int ngrp_row = p.ld / p.group;
    const float ro = valid ? p.row_out[row] : 1.f;
    const float ri = valid ? p.row_in[row] : 1.f;
    float r2 = 0.f, s2 = 0.f;
    for (int c0 = 0; c0 < 128; c0 += p.group) {
      const int col = col0 + c0;
      if (col >= g.N) break;
      const long long off = (long long)(valid ? row : 0) * p.ld + col;
      const long long goff = (long long)(valid ? row : 0) * ngrp_row + col / p.group;
      ProjRow r;
      r.V = p.V + off;
      r.sig = p.sig + col;
      r.rsig = p.rsig + col;
      r.hd = p.hd + col;
      r.codes = p.codes + off;
      r.phi = plane0_at(ENC, p.p_hi, valid ? row : 0, p.ld, col);
      r.plo = plane1_at(ENC, p.p_lo, valid ? row : 0, p.ld, col);
      r.scale = p.scale + goff;
      r.zero = p.zero + goff;
      r.wdump = p.wdump ? p.wdump + off : nullptr;
      r.rs = ri;
      r.flag = p.flag;
      r.vs = p.vs;
      r.fit_w = p.fit_w;
      r.valid = valid;
      r.grid_out = true;
      r.codes_in = nullptr;  // read from global memory (COLS_SMEM = false)
      r.scale_in = nullptr;
      r.zero_in = nullptr;
      // W~ = Q T: the accumulator carries the operands' scales (exact powers of two)
      auto loadw = [&](int c, float (&w)[32]) {
        tmem_ld32(taddr + c0 + c, w);
#pragma unroll
        for (int k = 0; k < 32; ++k) w[k] = __fmul_rn(w[k], ro);
      };
      auto loadv = [&](int c, float (&v)[8]) {
        if (valid) ld_v8f(r.V + c, v);
      };
      project_group<MODE, ENC>(loadw, loadv, r, p.group, p.L, r2, s2);
    }
    r2 = warp_sum(r2);
    s2 = warp_sum(s2);
    if ((rit & 31) == 0) {
      const int tile = (col0 >> 7) * g.tiles_m + tm;  // 128 x 128 tile of the output
      p.part[(tile * 4 + (rit >> 5)) * 2 + 0] = r2;
      p.part[(tile * 4 + (rit >> 5)) * 2 + 1] = s2;
    }
  }
};

// Objective: sum_k lambda_k acc_{jk}^2 per tile and warp.
struct EpiObjective {
  static constexpr bool FROM_TMEM = false;
  struct Params {
    const float* lam;
    const float* row_out;  // per-row factor that unscales the GEMM result
    float* part;           // [128-row tiles x 128-column tiles][4]
  };
  __device__ static void apply_regs(const Params& p, const GemmGeom& g, const float (&acc)[128],
                                    int tm, int, int, int rit, int col0) {
    const int row = tm * 128 + rit;
    float s = 0.f;
    if (row < g.M) {
      const float ro = p.row_out[row];
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        if (col0 + c < g.N) {
          float l[8];
          load8_ro(p.lam + col0 + c, l);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float a = __fmul_rn(acc[c + k], ro);
            s += l[k] * a * a;
          }
        }
      }
    }
    s = warp_sum(s);
    if ((rit & 31) == 0) p.part[((col0 >> 7) * g.tiles_m + tm) * 4 + (rit >> 5)] = s;
  }
};

}  // namespace admmq
