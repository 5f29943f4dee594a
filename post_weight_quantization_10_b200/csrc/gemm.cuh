// gemm.cuh -- persistent tcgen05 GEMM engine for sm_100a.
//
// D[M x N] = A[M x K] * B[K x N] with operands staged in shared memory by TMA
// (128-byte swizzle, every CTA loading its own tiles) and fp32 accumulation.  Operands are bf16
// (kind::f16) or tf32 held in fp32 words (kind::tf32); a shared-memory row is
// always 128 bytes (64 bf16 or 32 fp32 along K) and one MMA consumes 32 bytes
// of K.  Split-precision products for fp32-accurate GEMMs (NPL = 2 planes):
//   3xTF32 (KIND_TF32): planes hi = tf32(x), lo = tf32(x - hi); each K step
//     issues A_hi*B_hi + A_hi*B_lo + A_lo*B_hi.
//   mixed (KIND_MIX): plane 0 holds hi = tf32(x); plane 1 holds bf16
//     correction rows, each 128-byte row covering the same 32 K-elements as
//     plane 0's row: [bf16(hi) x32 | bf16(lo) x32] for A and
//     [bf16(lo) x32 | bf16(hi) x32] for B, lo = x - hi.  Each K step issues
//     one tf32 MMA on plane 0 and one bf16 MMA on plane 1, whose K = 16 runs
//     over hi(A).lo(B) and lo(A).hi(B): the same three terms in ~2/3 of the
//     tensor time, the correction terms carried to bf16 precision.
//   fp16 x3 (KIND_F16X3): planes hi = fp16(x s), lo = fp16(x s - hi) for a
//     power-of-two scale s chosen by the encoder (fp16's range is narrow);
//     each K step issues hi*hi + hi*lo + lo*hi as three kind::f16 MMAs.
//     fp16 products are exact in the fp32 accumulator and hi + lo carries 22
//     bits, as in 3xTF32, at the full 16-bit rate: 3 bf16-MMA units of
//     tensor time per product against 4 for the mixed split.
//
// Promoted accumulation.  The tensor core adds every MMA into its fp32
// accumulator with a small one-sided rounding error, so a long K sum drifts by
// a relative amount proportional to the number of MMAs (measured 2.9e-5 for
// K = 4096 with 3xTF32).  The MMA therefore writes each chunk of KC k-blocks
// into a fresh tensor-memory slot (a ring of two 256-column slots), and the
// consumer warps add the chunks into fp32 registers with round-to-nearest:
// the drift is bounded by one chunk.
//
// Tiles are 128 (CTA pairs: 256) rows x 256 columns.  Warp roles (320
// threads, one CTA per SM, 512 tensor-memory columns):
//   warp 0      TMA producer (one thread)
//   warp 1      tensor-memory owner and MMA issuer (one thread)
//   warps 2..9  two consumer warpgroups: thread = accumulator row, each
//               warpgroup 128 of the tile's 256 columns, summed in registers;
//               the epilogue runs from those registers (apply_regs) or, for
//               an epilogue that reads the tile twice (FROM_TMEM), from the
//               last chunk's slot, where the sum is written back and which
//               is released only afterwards (apply_tmem).
// CTA pairs (PAIR): a cluster of two CTAs runs 2-SM MMAs (cta_group::2) of
// 256 x 256: each CTA stages its 128 A rows and 128 of the 256 B rows; the
// leader (rank 0) issues the MMAs and commits to the barriers of both CTAs;
// both CTAs' TMA loads count on the leader's stage barrier; consumers release
// ring slots to the leader with remote arrivals.
// What a unit is comes from the Work policy: OneGemm (below) runs the (tile,
// k-split) units of one GEMM with one epilogue, dealt to CTAs (or pairs)
// round-robin.  A policy may also chain several GEMMs in one launch, with
// units whose operands are produced by earlier units of the same launch
// (ready counters, see ptx.cuh: wait_counter); such a policy deals its units
// dynamically (DYNAMIC): the pair leader's producer takes the next unit from
// a global ticket counter and passes it to its roles and to its pair member
// through a four-entry ring in shared memory.  A unit is then only ever taken
// by a running CTA, after every unit with a smaller index, so units waiting
// on smaller ones always make progress.  Every wait is bounded.
#pragma once
#include "ptx.cuh"

namespace admmq {

struct GemmGeom {
  int M, N, K;        // output rows / columns, reduction length
  int tiles_m;        // 128-row output tiles (counted up to whole units)
  int tiles_n;        // 256-column output tiles
  int tiles_mu;       // unit rows: 128-row tiles, or 256-row tile pairs
  int splits;         // k-splits per tile (units = tiles * splits)
  int kblocks;        // ceil(K / BK)
  int triangle;       // 1: only tiles that meet the upper triangle (i <= j)
  int tiles;          // number of tiles visited
  int units;          // tiles * splits
  int band;           // tile rows per band of the visiting order (L2 reuse)
  int* status;        // kernel status word (device)
};

// Operand kinds: KIND_BF16 / KIND_TF32 are the instruction-descriptor formats
// of plain products.  KIND_MIX is the split-precision product with one tf32
// plane and one bf16 correction plane per operand (see above).
enum { KIND_BF16 = 1, KIND_TF32 = 2, KIND_MIX = 3, KIND_F16X3 = 4 };

template <int KIND_, int NPL_, bool A_MN_, bool B_MN_, int STAGES_, int KC_, bool PAIR_>
struct GemmCfg {
  static constexpr int KIND = KIND_;
  static constexpr int ELEM = (KIND == KIND_BF16 || KIND == KIND_F16X3) ? 2 : 4;  // bytes per (plane-0) element
  static constexpr int BM = 128, BN = 256, BK = 128 / ELEM, NPL = NPL_, STAGES = STAGES_;
  static constexpr int UK = 32 / ELEM;                     // K per MMA instruction
  static constexpr int KC = KC_;                           // k-blocks per promoted chunk
  static constexpr bool A_MN = A_MN_, B_MN = B_MN_;
  static constexpr bool PAIR = PAIR_;
  static constexpr int UNIT_M = PAIR ? 2 * BM : BM;   // output rows per work unit
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;   // B rows staged per CTA
  static constexpr int A_PLANE = BM * 128;  // bytes per operand plane per stage
  static constexpr int B_PLANE = B_ROWS * 128;
  static constexpr int STAGE = NPL * (A_PLANE + B_PLANE);
  static constexpr int RING = 2;                 // 256-column chunk slots in tensor memory
  static constexpr int TMEM_COLS = RING * BN;    // 512
  static constexpr int THREADS = 320;
  // mbarriers (stages, ring slots, drain, unit ring), then tensor-memory
  // address, abort flag, 2 spare words, the four unit-completion counters of
  // the consumer warps and the four unit-ring entries
  static constexpr int UNIT_RING = 4;
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * RING + 1 + 2 * UNIT_RING) + 48;
  // readers that release a unit-ring entry: the MMA issuer and the eight
  // consumer warps of the leader, and the producer and eight consumer warps of
  // its pair member
  static constexpr int RING_READERS = PAIR ? 18 : 9;
  // arrivals that release a ring slot: every consumer thread of the CTA, or
  // one per consumer warp of both CTAs of a pair
  static constexpr int SLOT_ARRIVALS = PAIR ? 16 : 256;
  static constexpr int SMEM = STAGES * STAGE + 1024 + BAR_BYTES;
  static_assert(!PAIR || (!A_MN && !B_MN), "CTA pairs: K-major operands");
  static_assert(KIND != KIND_MIX || (NPL == 2 && !A_MN && !B_MN), "mixed split: two K-major planes");
  // products per K step: 3xTF32 / fp16 x3 (hi.hi, hi.lo, lo.hi), mixed (tf32
  // hi.hi + one bf16 product over the [hi|lo] x [lo|hi] correction row), or one
  static constexpr int PRODUCTS = KIND == KIND_MIX ? 2 : (NPL == 2 ? 3 : 1);
  static_assert(KIND != KIND_F16X3 || NPL == 2, "fp16 x3: two planes");
  static_assert(SMEM <= 232448, "shared memory budget");
  // instruction-descriptor A/B format: kind::f16 takes 0 = f16, 1 = bf16;
  // kind::tf32 takes 2
  static constexpr uint32_t FMT = KIND == KIND_F16X3 ? 0u : (KIND == KIND_BF16 ? 1u : 2u);
};

// Unit -> (tile row, tile column, k-block range).  Splits are the outer index
// so that CTAs running at the same time work on the same k-range of different
// tiles.  Full grids are visited in bands of `band` unit rows, column by
// column inside a band, so that the tiles in flight share A rows and B
// columns in L2.  Triangle mode (square Gram) visits the 128-row tiles that
// meet the upper triangle, column by column.
template <int BM, int BN>
__device__ __forceinline__ void decode_unit(const GemmGeom& g, int u, int& tm, int& tn, int& split,
                                            int& kb0, int& kb1) {
  split = u / g.tiles;
  int t = u - split * g.tiles;
  if (!g.triangle) {
    const int b = t / (g.band * g.tiles_n);
    const int rows = min(g.band, g.tiles_mu - b * g.band);
    const int r = t - b * g.band * g.tiles_n;
    tn = r / rows;
    tm = b * g.band + (r - tn * rows);
  } else {
    tn = 0;
    for (;;) {
      int cnt = ((tn + 1) * BN + BM - 1) / BM;
      if (cnt > g.tiles_mu) cnt = g.tiles_mu;
      if (t < cnt) break;
      t -= cnt;
      ++tn;
    }
    tm = t;
  }
  kb0 = (int)(((long long)split * g.kblocks) / g.splits);
  kb1 = (int)(((long long)(split + 1) * g.kblocks) / g.splits);
}

// One work unit: which GEMM of the launch (phase), which iteration (t), the
// output tile and the k-block range.
struct Unit {
  int phase, t, tm, tn, split, kb0, kb1;
};

// Work policy of a plain GEMM: the (tile, k-split) units of one geometry, one
// pair of operand maps per operand (planes 0 and 1), one epilogue.
template <class Epi>
struct OneGemm {
  struct Args {
    CUtensorMap a[2], b[2];
    GemmGeom g;
    typename Epi::Params ep;
  };
  static constexpr bool SIGNALS = false;
  static constexpr bool DYNAMIC = false;
  __device__ static int units(const Args& x) { return x.g.units; }
  template <class Cfg>
  __device__ static void decode(const Args& x, int u, Unit& w) {
    w.phase = 0;
    w.t = 0;
    decode_unit<Cfg::BM, Cfg::BN>(x.g, u, w.tm, w.tn, w.split, w.kb0, w.kb1);
  }
  __device__ static const CUtensorMap* map_a(const Args& x, const Unit&, int p) { return &x.a[p]; }
  __device__ static const CUtensorMap* map_b(const Args& x, const Unit&, int p) { return &x.b[p]; }
  __device__ static void prefetch(const Args& x, int npl) {
    for (int p = 0; p < npl; ++p) {
      prefetch_tmap(&x.a[p]);
      prefetch_tmap(&x.b[p]);
    }
  }
  __device__ static bool ready(const Args&, const Unit&, volatile int*) { return true; }
  __device__ static bool from_tmem(const Unit&) { return Epi::FROM_TMEM; }
  __device__ static void epi_regs(const Args& x, const Unit& w, const float (&acc)[128], int tile_m,
                                  int rit, int col0) {
    if constexpr (!Epi::FROM_TMEM) Epi::apply_regs(x.ep, x.g, acc, tile_m, w.tn, w.split, rit, col0);
  }
  __device__ static void epi_tmem(const Args& x, const Unit&, uint32_t ta, int tile_m, int rit,
                                  int col0) {
    if constexpr (Epi::FROM_TMEM) Epi::apply_tmem(x.ep, x.g, ta, tile_m, rit, col0);
  }
  __device__ static int* done_counter(const Args&, const Unit&) { return nullptr; }
};

template <class Cfg, class Work>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    k_gemm(const __grid_constant__ typename Work::Args args) {
  constexpr int BM = Cfg::BM, BN = Cfg::BN, STAGES = Cfg::STAGES, NPL = Cfg::NPL, KC = Cfg::KC;
  const GemmGeom& g = args.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  // Ring-slot barriers: both consumer warpgroups drain every chunk.
  constexpr int R = Cfg::RING;
  uint64_t* rfull = bars + 2 * STAGES;  // [slot]: slot holds a finished chunk
  uint64_t* rempty = rfull + R;         // [slot]: slot drained by its consumers
  uint64_t* drain = rempty + R;
  constexpr int UR = Cfg::UNIT_RING;
  uint64_t* ufull = drain + 1;          // [UR]: unit-ring entry written
  uint64_t* uempty = ufull + UR;        // [UR]: entry read by every reader (leader's)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(uempty + UR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* epi_count = reinterpret_cast<int*>(tmem_slot + 4);  // [4], by unit sequence number & 3
  volatile int* unit_ring = reinterpret_cast<volatile int*>(tmem_slot + 8);  // [UR]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA pairs: rank in the cluster (0 = leader, issues the MMAs); work units
  // are dealt per cluster.
  const uint32_t rank = Cfg::PAIR ? cluster_rank() : 0u;
  const int unit0 = Cfg::PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int unit_step = Cfg::PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int nunits = Work::units(args);
  constexpr bool DYN = Work::DYNAMIC;
  const bool leader = !Cfg::PAIR || rank == 0;
  // Dynamic dealing, reader side: the unit of this CTA's seq-th entry, -1 if
  // the wait gave up.  Every lane of the calling warp calls it (or the one
  // thread of a single-thread role); one arrival per warp releases the entry
  // on the leader's barrier.
  auto take_unit = [&](int seq, bool single) -> int {
    const int e = seq % UR;
    const uint32_t par = (uint32_t)(seq / UR) & 1u;
    const bool got = leader ? mbar_wait(smem_u32(&ufull[e]), par, abort_flag, g.status)
                            : mbar_wait_cluster(smem_u32(&ufull[e]), par, abort_flag, g.status);
    if (single ? !got : !__all_sync(0xffffffffu, got)) return -1;
    const int u = unit_ring[e];
    if (!single) __syncwarp();
    if (single || (threadIdx.x & 31) == 0) {
      if (leader)
        mbar_arrive(smem_u32(&uempty[e]));
      else
        mbar_arrive_cluster(cluster_addr(smem_u32(&uempty[e]), 0));
    }
    return u;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < R; ++a) {
      mbar_init(smem_u32(&rfull[a]), 1);
      mbar_init(smem_u32(&rempty[a]), Cfg::SLOT_ARRIVALS);
    }
    mbar_init(smem_u32(drain), 1);
    for (int e = 0; e < UR; ++e) {
      mbar_init(smem_u32(&ufull[e]), 1);
      mbar_init(smem_u32(&uempty[e]), Cfg::RING_READERS);
    }
    *abort_flag = 0;
    for (int k = 0; k < 4; ++k) epi_count[k] = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) Work::prefetch(args, NPL);
  if (warp == 1) {
    if (Cfg::PAIR)
      tmem_alloc_pair(smem_u32(tmem_slot), Cfg::TMEM_COLS);
    else
      tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
  }
  __syncthreads();
  if (Cfg::PAIR) cluster_sync();  // both CTAs' barriers exist before any remote use
  tc_fence_after();

  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      if constexpr (DYN) {
        if (blockIdx.x == 0) Work::begin(args);
      }
      for (int seq = 0; ok; ++seq) {
        int u = unit0 + seq * unit_step;
        if constexpr (DYN) {
          if (leader) {
            // take a ticket and pass it to this CTA's roles and to the pair member
            const int e = seq % UR;
            if (seq >= UR && !mbar_wait_cluster(smem_u32(&uempty[e]), (uint32_t)(seq / UR - 1) & 1u,
                                                abort_flag, g.status)) {
              ok = false;
              break;
            }
            u = Work::take_ticket(args);
            if (u > nunits) u = nunits;
            unit_ring[e] = u;
            mbar_arrive(smem_u32(&ufull[e]));
            if (Cfg::PAIR) {
              st_cluster_u32(cluster_addr(smem_u32((const void*)&unit_ring[e]), 1), (uint32_t)u);
              mbar_arrive_cluster(cluster_addr(smem_u32(&ufull[e]), 1));
            }
          } else {
            u = take_unit(seq, true);
            if (u < 0) {
              ok = false;
              break;
            }
          }
        }
        if (u >= nunits) break;
        Unit w;
        Work::template decode<Cfg>(args, u, w);
        // operands written earlier in this launch are published first
        if (!Work::ready(args, w, abort_flag)) {
          ok = false;
          break;
        }
        const int a_row = w.tm * Cfg::UNIT_M + (int)rank * BM;        // this CTA's A rows
        const int b_row = w.tn * BN + (int)rank * Cfg::B_ROWS;        // this CTA's B rows
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, abort_flag, g.status)) {
            ok = false;
            break;
          }
          // A pair's loads all count on the leader's barrier, which expects
          // the bytes of both CTAs.
          uint32_t fb = smem_u32(&full[s]);
          if (Cfg::PAIR) {
            if (rank == 0) mbar_arrive_expect_tx(fb, 2 * Cfg::STAGE);
            fb = cluster_addr(fb, 0);
          } else {
            mbar_arrive_expect_tx(fb, Cfg::STAGE);
          }
          const uint32_t st = smem_u32(smem + s * Cfg::STAGE);
          const int k0 = kb * Cfg::BK;
#pragma unroll
          for (int p = 0; p < NPL; ++p) {
            const uint32_t dA = st + p * Cfg::A_PLANE;
            const CUtensorMap* ma = Work::map_a(args, w, p);
            if (!Cfg::A_MN) {
              // a mixed correction plane holds two bf16 per K-element
              const int xa = (Cfg::KIND == KIND_MIX && p == 1) ? 2 * k0 : k0;
              if (Cfg::PAIR)
                tma_load_2d_pair(dA, ma, xa, a_row, fb);
              else
                tma_load_2d(dA, ma, xa, a_row, fb);
            } else {
#pragma unroll
              for (int b = 0; b < BM / (128 / Cfg::ELEM); ++b)
                tma_load_2d(dA + b * Cfg::BK * 128, ma, a_row + (128 / Cfg::ELEM) * b, k0, fb);
            }
          }
#pragma unroll
          for (int p = 0; p < NPL; ++p) {
            const uint32_t dB = st + NPL * Cfg::A_PLANE + p * Cfg::B_PLANE;
            const CUtensorMap* mb = Work::map_b(args, w, p);
            if (!Cfg::B_MN) {
              const int xb = (Cfg::KIND == KIND_MIX && p == 1) ? 2 * k0 : k0;
              if (Cfg::PAIR)
                tma_load_2d_pair(dB, mb, xb, b_row, fb);
              else
                tma_load_2d(dB, mb, xb, b_row, fb);
            } else {
#pragma unroll
              for (int b = 0; b < BN / (128 / Cfg::ELEM); ++b)
                tma_load_2d(dB + b * Cfg::BK * 128, mb, w.tn * BN + (128 / Cfg::ELEM) * b, k0, fb);
            }
          }
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA retires.  A
        // pair member's copies count on the leader's barriers: it waits a
        // fixed ~1 ms instead.
        if (!Cfg::PAIR || rank == 0) {
          for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
            mbar_wait_drain(smem_u32(&full[j % STAGES]), (uint32_t)(j / STAGES) & 1u);
        } else {
          const long long t0 = clock64();
          while (clock64() - t0 < 2000000LL) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // (a pair's MMAs, 256 rows of the unit, are issued by its leader alone)
    if (lane == 0 && (!Cfg::PAIR || rank == 0)) {
      constexpr uint32_t IDESC = idesc_f32acc(Cfg::FMT, Cfg::UNIT_M, BN, Cfg::A_MN, Cfg::B_MN);
      constexpr uint32_t IDESC16 = idesc_f32acc(KIND_BF16, Cfg::UNIT_M, BN, Cfg::A_MN, Cfg::B_MN);
      // a completed group of MMAs is announced on the barrier at the same
      // offset in each CTA of the pair (or in this CTA)
      auto commit_all = [&](uint64_t* bar) {
        if (Cfg::PAIR) {
          mma_commit_pair(cluster_addr(smem_u32(bar), 0));
          mma_commit_pair(cluster_addr(smem_u32(bar), 1));
        } else {
          mma_commit(smem_u32(bar));
        }
      };
      // MN-major: blocks of 128 bytes along MN, BK K-rows each, LBO apart
      constexpr uint32_t LBO_A = Cfg::A_MN ? Cfg::BK * 128 : 16;
      constexpr uint32_t LBO_B = Cfg::B_MN ? Cfg::BK * 128 : 16;
      constexpr int kStageStep = Cfg::STAGE >> 4, kAPlane = Cfg::A_PLANE >> 4;
      constexpr int kBPlane = Cfg::B_PLANE >> 4;
      constexpr int kKStepA = (Cfg::A_MN ? Cfg::UK * 128 : 32) >> 4;
      constexpr int kKStepB = (Cfg::B_MN ? Cfg::UK * 128 : 32) >> 4;
      const uint64_t descA0 = smem_desc_sw128(smem_u32(smem), LBO_A, 1024);
      const uint64_t descB0 = smem_desc_sw128(smem_u32(smem + NPL * Cfg::A_PLANE), LBO_B, 1024);
      int it = 0;
      uint32_t q = 0;  // chunks issued: chunk q goes to slot q % R, use q / R of it
      bool ok = true;
      for (int seq = 0; ok; ++seq) {
        int u = unit0 + seq * unit_step;
        if constexpr (DYN) {
          u = take_unit(seq, true);
          if (u < 0) {
            ok = false;
            break;
          }
        }
        if (u >= nunits) break;
        Unit w;
        Work::template decode<Cfg>(args, u, w);
        const int kb0 = w.kb0, kb1 = w.kb1;
        for (int c0 = kb0; c0 < kb1 && ok; c0 += KC, ++q) {
          const int c1 = min(c0 + KC, kb1);
          const uint32_t slot = q % R;
          if (q >= (uint32_t)R) {
            // wait until the slot's previous chunk has been drained
            if (!mbar_wait(smem_u32(&rempty[slot]), (q / R - 1u) & 1u, abort_flag, g.status)) {
              ok = false;
              break;
            }
          }
          tc_fence_after();
          const uint32_t dt = tmem_base + slot * BN;
          for (int kb = c0; kb < c1; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
            if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag, g.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // descriptors of this stage: the start-address field counts
            // 16-byte units, so planes, stages and K steps are plain adds
            const uint64_t a0 = descA0 + (uint64_t)s * kStageStep;
            const uint64_t b0 = descB0 + (uint64_t)s * kStageStep;
            const uint32_t acc0 = (kb > c0) ? 1u : 0u;
#pragma unroll
            for (int kk = 0; kk < Cfg::BK / Cfg::UK; ++kk) {
#pragma unroll
              for (int pr = 0; pr < Cfg::PRODUCTS; ++pr) {
                // 3xTF32: (hi,hi), (hi,lo), (lo,hi); mixed: (0,0) tf32, (1,1) bf16
                const int pa = Cfg::KIND == KIND_MIX ? pr : ((pr == 2) ? 1 : 0);
                const int pb = Cfg::KIND == KIND_MIX ? pr : ((pr == 1) ? 1 : 0);
                const uint64_t ad = a0 + (uint64_t)(pa * kAPlane + kk * kKStepA);
                const uint64_t bd = b0 + (uint64_t)(pb * kBPlane + kk * kKStepB);
                const uint32_t accum = (kk > 0 || pr > 0) ? 1u : acc0;
                // a kind::f16 MMA (bf16 or fp16 operands) or a kind::tf32 one
                const bool b16 = Cfg::KIND == KIND_BF16 || Cfg::KIND == KIND_F16X3 ||
                                 (Cfg::KIND == KIND_MIX && pr == 1);
                const uint32_t id = Cfg::KIND == KIND_MIX && pr == 1 ? IDESC16 : IDESC;
                if (Cfg::PAIR) {
                  if (b16)
                    mma_f16_pair(dt, ad, bd, id, accum);
                  else
                    mma_tf32_pair(dt, ad, bd, id, accum);
                } else {
                  if (b16)
                    mma_f16(dt, ad, bd, id, accum);
                  else
                    mma_tf32(dt, ad, bd, id, accum);
                }
              }
            }
            commit_all(&empty[s]);
          }
          if (!ok) break;
          commit_all(&rfull[slot]);
        }
      }
      // Every MMA issued above is complete once this arrives.
      if (Cfg::PAIR)
        mma_commit_pair(cluster_addr(smem_u32(drain), 0));
      else
        mma_commit(smem_u32(drain));
      mbar_wait_drain(smem_u32(drain), 0);
    }
  } else {
    // ---------------------------------------------------------- consumers
    const int wg = (warp - 2) >> 2;  // consumer warpgroup 0 or 1: columns 128 wg ..
    const int qtr = warp & 3;        // tensor-memory lane quarter this warp may access
    const uint32_t lane_off = (uint32_t)(qtr * 32) << 16;
    const uint32_t col_off = (uint32_t)(wg * 128);
    uint32_t q = 0;  // chunks consumed: chunk q is use q / R of slot q % R
    bool ok = true;
    // a pair member drains its slots for the leader's MMA issuer
    const uint32_t rempty_leader = Cfg::PAIR ? cluster_addr(smem_u32(rempty), 0) : 0u;
    // releases ring slot `slot` for the MMA issuer (of this CTA or of the pair)
    auto release = [&](uint32_t slot) {
      if (Cfg::PAIR) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(rempty_leader + 8u * slot);
      } else {
        mbar_arrive(smem_u32(&rempty[slot]));
      }
    };
    for (int seq = 0; ok; ++seq) {  // seq: units this CTA has taken
      int u = unit0 + seq * unit_step;
      if constexpr (DYN) {
        u = take_unit(seq, false);
        if (u < 0) {
          ok = false;
          break;
        }
      }
      if (u >= nunits) break;
      Unit w;
      Work::template decode<Cfg>(args, u, w);
      const int kb0 = w.kb0, kb1 = w.kb1;
      const bool from_tmem = Work::from_tmem(w);
      const int tile_m = Cfg::PAIR ? 2 * w.tm + (int)rank : w.tm;  // this CTA's 128-row tile
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
      uint32_t kept = 0;
      for (int c0 = kb0; c0 < kb1; c0 += KC, ++q) {
        const uint32_t slot = q % R;
        const bool got = mbar_wait(smem_u32(&rfull[slot]), (q / R) & 1u, abort_flag, g.status);
        if (!__all_sync(0xffffffffu, got)) {  // tcgen05.ld needs all 32 lanes
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem_base + lane_off + slot * BN + col_off;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float v[16];
          tmem_ld16(ta + 16 * j, v);
#pragma unroll
          for (int k = 0; k < 16; ++k) acc[16 * j + k] += v[k];
        }
        tc_fence_before();
        // An epilogue that reads the tile from tensor memory keeps the last
        // chunk's slot: the summed accumulator goes back into it below.
        if (from_tmem && c0 + KC >= kb1)
          kept = slot;
        else
          release(slot);
      }
      if (!ok) continue;
      const int col0 = w.tn * BN + wg * 128;
      if (from_tmem) {
        const uint32_t ta = tmem_base + lane_off + kept * BN + col_off;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float v[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = acc[32 * j + k];
          tmem_st32(ta + 32 * j, v);
        }
        Work::epi_tmem(args, w, ta, tile_m, qtr * 32 + lane, col0);
        tc_fence_before();
        release(kept);
      } else {
        Work::epi_regs(args, w, acc, tile_m, qtr * 32 + lane, col0);
      }
      if constexpr (Work::SIGNALS) {
        // Publish this unit's stores: every thread makes them visible to the
        // GPU (and to TMA reads); the last of the CTA's eight consumer warps
        // to finish the unit adds one to its ready counter.  Warps never
        // drift four units apart (each chunk's slot is released by all of
        // them), so four counters indexed by the unit's sequence number keep
        // the arrivals of different units apart.
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) {
          const int old = atom_add_acq_rel_cta(smem_u32(&epi_count[seq & 3]), 1);
          if ((old & 7) == 7) red_release_gpu_add(Work::done_counter(args, w), 1);
        }
      }
    }
  }
  __syncthreads();
  if (Cfg::PAIR) cluster_sync();  // the peer's last remote arrivals have landed
  if (warp == 1) {
    tc_fence_after();
    if (Cfg::PAIR)
      tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace admmq
