// admm_loop.cuh -- ADMM-Q iterations as one persistent launch of the engine.
//
// Every step of an iteration acts on rows ("ADMM-Q: An Improved Hessian-based
// Weight Quantizer ...", Methodology section 2: W-update, D-update, dual
// update): row block r of T needs only row block r of P (GEMM 1); row block r
// of W~ needs only row block r of T (GEMM 2), whose epilogue refreshes row
// block r of P, V~ and the codes.  So the units of GEMM 1 and GEMM 2 of
// every iteration share one launch, ordered (iteration, GEMM, tile) and
// dealt to the CTA pairs in that order from a ticket counter: the units in
// flight are always a narrow window of consecutive indices, whose tiles share
// their operand panels in L2, however long the launch.  Before loading, a
// unit's producer waits until the row block it reads is complete:
//   GEMM 2 of iteration i, row block r: every GEMM-1 tile of (i, r) is done;
//   GEMM 1 of iteration i > 0, row block r: every GEMM-2 tile of (i - 1, r).
// The same waits cover the overwrites: GEMM 1 of i rewrites the T that GEMM 2
// of i - 1 read, GEMM 2 of i the P that GEMM 1 of i read.
// Every dependency has a smaller unit index and a unit is only taken by a
// running pair after every smaller one, so the lowest unfinished unit is
// always held by a running pair and can proceed, however many pairs are
// resident; the waits are bounded all the same.  The arithmetic of each unit
// is that of the separate GEMM launches, so both schedules give the same bits.
#pragma once
#include "gemm.cuh"

namespace admmq {

template <class Epi1, class Epi2>
struct AdmmLoop {
  static_assert(!Epi1::FROM_TMEM && Epi2::FROM_TMEM, "GEMM 1 from registers, GEMM 2 from tensor memory");
  struct Args {
    CUtensorMap a[2][2], b[2][2];  // [GEMM][plane]: GEMM 1 A = P, B = E; GEMM 2 A = T, B = Q
    GemmGeom g;                    // one GEMM's geometry (M = d_out, N = K = d_in)
    typename Epi1::Params p1;      // rho taken per unit from rho[t]
    typename Epi2::Params p2;      // part taken per unit: part0 + t * part_stride
    const float* rho;              // [iterations] rho_t
    const float* vscale;           // [iterations] dual rescaling after iteration t
    float* part0;
    long long part_stride;
    int* ready;                    // [2][tiles_mu] finished CTA tiles per row block
    int base;                      // iterations already counted in `ready`
    int* ticket;                   // next unit to deal, zero before the launch
    int* ticket_next;              // the next launch's counter, zeroed by this one
    int ctas;                      // CTAs per unit (2 for CTA pairs)
    int t0, count;
  };
  static constexpr bool SIGNALS = true;
  static constexpr bool DYNAMIC = true;
  __device__ static int take_ticket(const Args& x) { return atomicAdd(x.ticket, 1); }
  // Launches alternate between two counters: each zeroes the other one for
  // the launch after it (which starts only once this one has ended), so an
  // aborted launch leaves no stale count behind.
  __device__ static void begin(const Args& x) { *x.ticket_next = 0; }
  __device__ static int units(const Args& x) { return x.count * 2 * x.g.units; }
  template <class Cfg>
  __device__ static void decode(const Args& x, int u, Unit& w) {
    const int U = x.g.units;
    const int i = u / (2 * U);
    const int r = u - i * 2 * U;
    w.phase = r >= U ? 1 : 0;
    w.t = x.t0 + i;
    decode_unit<Cfg::BM, Cfg::BN>(x.g, r - w.phase * U, w.tm, w.tn, w.split, w.kb0, w.kb1);
  }
  __device__ static const CUtensorMap* map_a(const Args& x, const Unit& w, int p) { return &x.a[w.phase][p]; }
  __device__ static const CUtensorMap* map_b(const Args& x, const Unit& w, int p) { return &x.b[w.phase][p]; }
  __device__ static void prefetch(const Args& x, int npl) {
    for (int ph = 0; ph < 2; ++ph)
      for (int p = 0; p < npl; ++p) {
        prefetch_tmap(&x.a[ph][p]);
        prefetch_tmap(&x.b[ph][p]);
      }
  }
  // Counters: [0][r] GEMM-1 tiles of row block r finished, [1][r] GEMM-2
  // tiles, counted over every iteration since they were zeroed (`base` of them
  // before this launch).
  __device__ static bool ready(const Args& x, const Unit& w, volatile int* abort_flag) {
    const int per = x.ctas * x.g.tiles_n;  // CTA tiles per row block and GEMM
    const int i = w.t - x.t0;
    if (w.phase == 0) {
      if (i == 0) return true;  // an earlier launch (or the setup) wrote P
      return wait_counter(x.ready + x.g.tiles_mu + w.tm, (x.base + i) * per, abort_flag, x.g.status);
    }
    return wait_counter(x.ready + w.tm, (x.base + i + 1) * per, abort_flag, x.g.status);
  }
  __device__ static bool from_tmem(const Unit& w) { return w.phase == 1; }
  __device__ static void epi_regs(const Args& x, const Unit& w, const float (&acc)[128], int tile_m,
                                  int rit, int col0) {
    typename Epi1::Params p = x.p1;
    p.rho = x.rho[w.t];
    Epi1::apply_regs(p, x.g, acc, tile_m, w.tn, w.split, rit, col0);
  }
  __device__ static void epi_tmem(const Args& x, const Unit& w, uint32_t ta, int tile_m, int rit,
                                  int col0) {
    typename Epi2::Params p = x.p2;
    p.part = x.part0 + (long long)w.t * x.part_stride;
    p.vs = x.vscale[w.t];
    Epi2::apply_tmem(p, x.g, ta, tile_m, rit, col0);
  }
  __device__ static int* done_counter(const Args& x, const Unit& w) {
    return x.ready + w.phase * x.g.tiles_mu + w.tm;
  }
};

}  // namespace admmq
