// Whole-token persistent decode kernel for batch 1 ("Density Field State Space
// Models", Section 4.1: the 48-layer forward of one decode token, here one launch).
//
// One CTA of 16 warps per SM for the whole token; CTAs form clusters of Q (<= 8).
//   * 15 compute warps run the layer's dependency chain;
//   * 1 copy warp streams each layer's per-CTA weight and state slices into shared
//     memory ahead of use, as bulk copies only (cp.async.bulk; the TMA engine moves
//     the bytes, so the copies neither stall the compute warps nor compete with their
//     shared-memory traffic).  Full/empty mbarrier pairs hand the buffers over.
// 16 warps, not 17, so that each thread may hold 128 registers.
//
// A layer is a chain of dependent steps whose cost is latency, not bytes (a layer
// moves 8 MB, 1.25 us of HBM time on the whole chip).  Measured on the B200: a
// grid-wide all-gather of tagged words costs ~1.5-1.8 us whether a CTA gathers a
// slice or the whole vector, and a cluster all-to-all ~0.6 us.  So:
//   * Two grid-wide exchanges per layer, the minimum for row-split projections (every
//     output row needs the whole input vector): the residual after out_proj and the
//     gated value after the SSM.  Every CTA gathers the WHOLE vector and prepares the
//     projection's activation itself (RMSNorm, fp16 rounding, six digit planes, exact
//     integer sum, max |x|): no slice all-gathers inside the cluster.
//   * Grid-wide words are "tagged words": 64-bit words holding 32 data bits and a
//     32-bit tag (launch epoch, layer, exchange kind), stored and polled without
//     fences; a word is valid exactly when its tag matches.  Each thread keeps all of
//     its words' loads in flight.  Producers also publish the fp64 sum of squares of
//     their values, so every consumer gets the RMSNorm without another reduction.
//   * Three cluster exchanges per layer, by st.async into every CTA of the cluster
//     (completion counted in bytes on the receiver's mbarrier), each overlapped with
//     tensor-core work: the int32 LoRA stage-1 partials of the in_proj (split over the
//     cluster by columns) behind the in_proj's shared tiles, the shared rows (B and C
//     after conv + SiLU, step sizes and decays, computed by every cluster for itself)
//     behind the z/x tiles, the out_proj's LoRA partials behind the out_proj tiles.
//
// Per layer (B = 1), CTA c of cluster k, rank r:
//   R   gather the residual (all D words) and the sums of squares
//   A   x = fp16(rmsnorm(res) w): six digit planes of all D columns, sum, max
//   L   int8 codes of slice r, LoRA partials of all rows -> the cluster
//   S   exact int8 scaffold MMA of this CTA's share of the cluster's shared tiles
//       (all B/C rows and the dt rows of the cluster's heads); LoRA stage 2, conv
//       step + SiLU (B/C), softplus and decay (dt) -> the cluster
//   Z   scaffold MMA of the z and x rows of its own SSM channels, LoRA stage 2, conv
//       step of its x channels, silu(z)
//   G   SSM update of its own state rows, g = y silu(z) and its sum of squares
//       published; gather all E gated values
//   A'L' the gated RMSNorm, codes and LoRA stage 1 of the out_proj
//   O   out_proj rows of its tiles added to the residual and published
// Final: gather the residual, final RMSNorm, stream this CTA's LM-head rows,
// publish (best logit, id); CTA 0 reduces to the greedy token.
//
// Every spin is bounded: a wait that gives up sets a status bit and an abort flag
// that makes every CTA leave the token early; all CTAs of a cluster meet at a
// final cluster barrier (after an abort, only once in-flight copies have had time
// to land), so none exits while another may still write into it.  A launch that
// finds the abort flag of an earlier call set does nothing (status value 1).
//
// Built with DFSSM_PHASE_TIMERS, thread 0 of every CTA adds the clock64 cycles of
// each phase (summed over the layers) into PParams::phase[CTA][slot].
#pragma once

#include "common.cuh"

// Built with DFSSM_NOINLINE, the large per-phase helpers are real calls (one copy
// of each in the kernel's code) instead of being inlined at every use.
#ifdef DFSSM_NOINLINE
#define DFSSM_BIG __device__ __noinline__
#else
#define DFSSM_BIG DFSSM_DEV
#endif

namespace dfssm {

constexpr int kMaxLayers = 64;
constexpr int kPWarps = 15;                       // compute warps
constexpr int kPThreads = 32 * kPWarps;           // compute threads
constexpr int kPBlock = kPThreads + 32;           // + the copy warp: 16 warps, 128 registers each
constexpr int kPMaxUnits = 3;                     // SSM row units (16 channels) per CTA
constexpr int kPMaxShared = 5;                    // shared (B/C, dt) tiles per CTA
constexpr int kPMaxInTiles = 9;                   // z, x and shared tiles per CTA
constexpr int kPMaxSharedTiles = 20;              // shared tiles of one cluster
constexpr int kPMaxSharedRows = 16 * kPMaxSharedTiles;
constexpr int kPMaxOutTiles = 2;                  // out_proj tiles per CTA
constexpr int kPMaxCluster = 8;
constexpr int kPMaxHeads = 4;                     // heads touched by one CTA's SSM rows
constexpr int kPMaxK = 4096;                      // largest d_model / d_inner of the token kernel
constexpr int kPSsmRows = (kPMaxUnits * 16 + kPWarps - 1) / kPWarps;   // SSM rows per compute warp
constexpr long long kSpinLimit = 1LL << 22;       // polls before a wait gives up (seconds)
constexpr int kHeadChunkRows = 15;                // LM-head fp16 rows per chunk: one per compute warp
constexpr int kHeadRingMax = 8;                   // LM-head chunk slots (all buffers free after the last layer)
constexpr int kPhaseSlots = 32;                   // phase-timer slots per CTA (the last counts calls)
constexpr int kPlanSMs = 256;                     // upper bound on CTAs of one launch (sizes the exchange scratch)

// tagged-word exchange kinds
enum { XR = 0, XG = 1, XHEAD = 2 };
// cluster exchanges (one mbarrier each, one phase per layer)
enum { EX_LIN = 0, EX_SH = 1, EX_LOUT = 2, EX_N = 3 };
// phase-timer slots (cycles of thread 0, summed over the layers)
enum {
  PH_GATHER_R = 0, PH_WAIT_AB, PH_PREP_IN, PH_LORA_IN, PH_MMA_SH, PH_WAIT_LIN, PH_SHARED, PH_MMA_ZX, PH_ZX_EPI,
  PH_WAIT_SH, PH_SSM, PH_GATHER_G, PH_WAIT_CD, PH_PREP_OUT, PH_LORA_OUT, PH_MMA_OUT, PH_WAIT_LOUT, PH_RESID,
  PH_HEAD, PH_HEAD_STREAM, PH_HEAD_ARG, PH_N   // LM head: gather + norm, row stream, argmax exchange
};

struct PLayer {
  const uint16_t* prenorm_w;
  const uint32_t* in_bits; const uint16_t* in_alpha; const int8_t* in_A; const uint16_t* in_sA;
  const int8_t* in_B; const uint16_t* in_sB;
  const uint16_t* conv_w; const uint16_t* conv_b;
  const float* dt_bias; const float* A_log; const float* D;
  const uint16_t* gnorm_w;
  const uint32_t* out_bits; const uint16_t* out_alpha; const int8_t* out_A; const uint16_t* out_sA;
  const int8_t* out_B; const uint16_t* out_sB;
  float* conv_state; float* ssm_state;
};

// Shared-memory layout (byte offsets), computed on the host for one shape.
struct PSmem {
  // layer group AB (refilled after the SSM phase; the LM-head ring reuses it)
  int in_tiles, in_bq, in_alpha, in_sb, convw_x, convb_x, cst_x;
  int sh_convw, sh_convb, sh_cst, a_in, prenorm, sa_in, hd_dtb, hd_alog, hd_d, state;
  int ab_end;
  // layer group CD (refilled after out_proj)
  int out_tiles, out_bq, out_alpha, out_sb, a_out, gnorm, sa_out;
  int cd_end;
  // working
  int vfull, planes, xs, xqs, rcv, yin, shr, shst, u, resown;
  int ring_end, head_slots;       // LM-head chunk slots [0, head_slots) tile [0, ring_end)
  int part, full, misc, lo2;
  int total;
};

struct __align__(16) PParams {
  // shape
  int n_layer, D, E, H, P, N, R, in_rows, C, vocab;
  int kg_in, kg_out;             // 256-column groups of the in/out projections
  int units, grid, Q;            // SSM row units (E/16), CTAs, CTAs per cluster
  int n_bc_tiles, dt_tile0;      // 2N/16 and first dt tile index
  int out_tiles;                 // D/16
  int SD, SE;                    // LoRA stage-1 column slices (D/Q, E/Q)
  int layer_mode;                // 1: residual in/out from `residual`, no embedding / head
  PSmem sm;
  // io
  const uint16_t* embed; const uint16_t* normf_w; const int32_t* tok_in; int32_t* tok_out; float* logits;
  const int8_t* embed_q;         // int8 per-row embedding (replaces embed when not null)
  const float* embed_s;          // its fp32 row scales
  float* residual;               // layer mode: [D] in/out
  // workspace
  unsigned* status;              // status word
  unsigned* ctl;                 // [0] launch epoch, [1] abort flag, [2] test: CTA + 1 that withholds its
                                 // layer-0 residual words, [3] test: polls before a wait gives up
  unsigned long long* x_r;       // D residual words
  unsigned long long* x_rs;      // 2 grid words: fp64 sum of squares of each CTA's residual rows
  unsigned long long* x_g;       // E gated-value words
  unsigned long long* x_gs;      // 2 grid words: fp64 sum of squares of each CTA's gated values
  unsigned long long* x_head;    // 2 grid words
  unsigned long long* phase;     // [grid][kPhaseSlots] phase cycles (timer builds), or null
  // diagnostics of the last layer (workspace regions of dfssm_ws_layout)
  uint16_t* d_x_in; int8_t* d_xq_in; float* d_sx_in; int* d_acc_in; double* d_u_in; int8_t* d_xd_in;
  int* d_xdsum_in; double* d_zx; double* d_xc; float* d_g; uint16_t* d_x_out; int8_t* d_xq_out;
  float* d_sx_out; int* d_acc_out; double* d_u_out; int8_t* d_xd_out; int* d_xdsum_out; float* d_res;
  PLayer L[kMaxLayers];
};

__host__ __device__ constexpr int ptake(int& off, int bytes) {
  const int at = off;
  off = (off + (bytes > 16 ? bytes : 16) + 15) & ~15;
  return at;
}

// Digit-plane stride of a K-column activation: K + 64 bytes, so that the 16-byte
// B-fragment loads of one quarter-warp (planes g, g + 1 at 16-byte offsets 0..48)
// fall in 8 distinct 16-byte bank groups.
__host__ __device__ constexpr int plane_stride(int K) { return K + 64; }

// Shared-memory plan of one shape (byte offsets) for clusters of Q CTAs holding at
// most U SSM units each; the host plans launches with the same function, and the
// compile-time shape below bakes its result into the code.
__host__ __device__ constexpr PSmem plan_smem(int D, int E, int H, int N, int R, int Q, int U) {
  PSmem m{};
  const int kg_in = D / kTileCols, kg_out = E / kTileCols;
  const int SD = D / Q, SE = E / Q;
  const int K = D > E ? D : E, Smax = SD > SE ? SD : SE, R4 = R > 4 ? R : 4, R1 = R > 1 ? R : 1;
  int off = 0;
  m.in_tiles = ptake(off, kPMaxInTiles * kg_in * 512);
  m.in_bq = ptake(off, kPMaxInTiles * 16 * R);
  m.in_alpha = ptake(off, kPMaxInTiles * 32);
  m.in_sb = ptake(off, kPMaxInTiles * 32);
  m.convw_x = ptake(off, kPMaxUnits * 128);
  m.convb_x = ptake(off, kPMaxUnits * 32);
  m.cst_x = ptake(off, 3 * kPMaxUnits * 64);
  m.sh_convw = ptake(off, kPMaxShared * 128);
  m.sh_convb = ptake(off, kPMaxShared * 32);
  m.sh_cst = ptake(off, 3 * kPMaxShared * 64);
  m.a_in = ptake(off, R * SD);
  m.prenorm = ptake(off, 2 * D);
  m.sa_in = ptake(off, 2 * R);
  m.hd_dtb = ptake(off, 4 * H);
  m.hd_alog = ptake(off, 4 * H);
  m.hd_d = ptake(off, 4 * H);
  m.state = ptake(off, U * 16 * N * 4);
  m.ab_end = off;
  m.out_tiles = ptake(off, kPMaxOutTiles * kg_out * 512);
  m.out_bq = ptake(off, kPMaxOutTiles * 16 * R);
  m.out_alpha = ptake(off, kPMaxOutTiles * 32);
  m.out_sb = ptake(off, kPMaxOutTiles * 32);
  m.a_out = ptake(off, R * SE);
  m.gnorm = ptake(off, 2 * E);
  m.sa_out = ptake(off, 2 * R);
  m.cd_end = off;
  m.vfull = ptake(off, 4 * K);
  m.planes = ptake(off, kDigits * plane_stride(K));
  m.xs = ptake(off, 2 * Smax);
  m.xqs = ptake(off, Smax);
  m.rcv = ptake(off, 2 * Q * 4 * R4);          // [2][Q][R]: in_proj and out_proj LoRA partials
  m.yin = ptake(off, kPMaxInTiles * 16 * 8);
  m.shr = ptake(off, 2 * kPMaxSharedRows * 8);
  m.shst = ptake(off, 3 * kPMaxShared * 16 * 4);
  m.u = ptake(off, 8 * R1);
  m.resown = ptake(off, kPMaxOutTiles * 16 * 4);
  // everything above is free once the last layer is done: the LM-head chunk ring
  // (grown to five chunks when that still leaves room for the rest)
  const int chunk = kHeadChunkRows * 2 * D;
  if (off < 5 * chunk && 5 * chunk + 4 * (2 * kPlanSMs + D) + 8 * 1024 <= 200 * 1024) off = 5 * chunk;
  m.ring_end = off;
  m.head_slots = off / chunk;
  if (m.head_slots > kHeadRingMax) m.head_slots = kHeadRingMax;
  m.part = ptake(off, 16 * 16 * kDigits * 4);
  m.full = ptake(off, 4 * (2 * kPlanSMs + D));
  m.misc = ptake(off, kPMaxInTiles * 16 * kDigits * 4);
  m.lo2 = ptake(off, kPMaxInTiles * 16 * 8);
  m.total = off;
  return m;
}

// Shapes: the kernel reads every size and shared-memory offset either from its
// parameters (any eligible shape) or from compile-time constants (the shape of the
// 48-layer, d_model 2048 model; address arithmetic then folds into immediates).
struct ShapeAny {
  static constexpr bool kConst = false;
  static constexpr int D = 0, E = 0, H = 0, P = 0, N = 0, R = 0, Q = 0, C = 0, kg_in = 0, kg_out = 0;
  static constexpr int SD = 0, SE = 0;
  static constexpr int units = 0, n_bc_tiles = 0, dt_tile0 = 0, out_tiles = 0;
  static constexpr PSmem kPlan{};
};
struct Shape2048 {
  static constexpr bool kConst = true;
  static constexpr int D = 2048, E = 4096, H = 64, P = 64, N = 128, R = 32, Q = 4, U = 2, C = E + 2 * N;
  static constexpr int kg_in = D / kTileCols, kg_out = E / kTileCols;
  static constexpr int SD = D / Q, SE = E / Q;
  static constexpr int units = E / 16, n_bc_tiles = 2 * N / 16, dt_tile0 = (2 * E + 2 * N) / 16, out_tiles = D / 16;
  static constexpr PSmem kPlan = plan_smem(D, E, H, N, R, Q, U);
};

// ------------------------------------------------------------------ primitives

DFSSM_DEV bool mbar_try_wait_cluster(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// 4 / 8 bytes into the shared memory of a CTA of the cluster (addresses from
// cluster_map), completion counted on that CTA's mbarrier.
DFSSM_DEV void st_async_b32(uint32_t dst, uint32_t v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
               :: "r"(dst), "r"(v), "r"(bar) : "memory");
}
DFSSM_DEV void st_async_b64(uint32_t dst, unsigned long long v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];"
               :: "r"(dst), "l"(v), "r"(bar) : "memory");
}
// Named barrier 1 over the CTA's 15 compute warps.
DFSSM_DEV void csync() { asm volatile("bar.sync 1, %0;" :: "n"(kPThreads) : "memory"); }
DFSSM_DEV bool csync_and(bool v) {
  unsigned r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r) : "r"(unsigned(v)), "n"(kPThreads) : "memory");
  return r != 0;
}

DFSSM_DEV void tw_put(unsigned long long* p, uint32_t v, uint32_t tag) {
  const unsigned long long w = (static_cast<unsigned long long>(tag) << 32) | v;
  asm volatile("st.volatile.global.u64 [%0], %1;" :: "l"(p), "l"(w) : "memory");
}
DFSSM_DEV void tw_put_f64(unsigned long long* p, double v, uint32_t tag) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(v));
  tw_put(p, uint32_t(b), tag);
  tw_put(p + 1, uint32_t(b >> 32), tag);
}
DFSSM_DEV unsigned long long tw_load(const unsigned long long* p) {
  unsigned long long w;
  asm volatile("ld.volatile.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}
DFSSM_DEV double f64_of(const uint32_t* w2) {
  return __longlong_as_double(static_cast<long long>((static_cast<unsigned long long>(w2[1]) << 32) | w2[0]));
}

DFSSM_DEV bool aborted(const unsigned* ctl) { return *reinterpret_cast<volatile const unsigned*>(ctl + 1) != 0; }

// Polls a wait makes before it gives up: control word 3 when a test sets it (so that a
// wait made to run out ends within milliseconds), else kSpinLimit.  Read only every
// 256 polls.
DFSSM_DEV long long spin_limit(const unsigned* ctl) {
  const unsigned v = *reinterpret_cast<volatile const unsigned*>(ctl + 3);
  return v ? static_cast<long long>(v) : kSpinLimit;
}

DFSSM_DEV void give_up(unsigned* status, unsigned* ctl, unsigned bit) {
  atomicOr(status, bit);
  atomicExch(ctl + 1, 1u);
}

// Compute warps: gather n1 tagged words from src1 into dst1 and n2 from src2 into
// dst2 (32-bit payloads).  Each thread keeps its (up to GW per pass) words' loads in
// flight and re-polls only the missing ones.  Returns false (after flagging) if a
// word did not arrive within the spin limit.
template <int GW>
DFSSM_BIG bool tw_gather(unsigned* status, unsigned* ctl, const unsigned long long* src1, int n1, uint32_t* dst1,
                         const unsigned long long* src2, int n2, uint32_t* dst2, uint32_t tag, unsigned bit) {
  bool ok = true;
  const int n = n1 + n2;
  for (int base = 0; base < n && ok; base += GW * kPThreads) {
    unsigned pending = 0;
#pragma unroll
    for (int i = 0; i < GW; ++i)
      if (base + i * kPThreads + int(threadIdx.x) < n) pending |= 1u << i;
    long long spins = 0;
    while (pending) {
      unsigned long long w[GW];
#pragma unroll
      for (int i = 0; i < GW; ++i) {
        const int idx = base + i * kPThreads + int(threadIdx.x);
        if (pending & (1u << i)) w[i] = tw_load(idx < n1 ? src1 + idx : src2 + (idx - n1));
      }
#pragma unroll
      for (int i = 0; i < GW; ++i) {
        const int idx = base + i * kPThreads + int(threadIdx.x);
        if ((pending & (1u << i)) && uint32_t(w[i] >> 32) == tag) {
          *(idx < n1 ? dst1 + idx : dst2 + (idx - n1)) = uint32_t(w[i]);
          pending &= ~(1u << i);
        }
      }
      if (pending) {
        if (((++spins & 255) == 0) && (spins > spin_limit(ctl) || aborted(ctl))) {
          give_up(status, ctl, bit);
          ok = false;
          break;
        }
        // a short pause between polls keeps the waiting CTAs' loads from crowding
        // the L2 that the producers are still writing through
        __nanosleep(64);
      }
    }
  }
  return csync_and(ok);
}

// Bounded wait by one thread.
DFSSM_DEV bool mbar_wait(unsigned* status, unsigned* ctl, uint64_t* bar, unsigned parity, unsigned bit) {
  long long spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if (((++spins & 255) == 0) && (spins > spin_limit(ctl) || aborted(ctl))) {
      give_up(status, ctl, bit);
      return false;
    }
  }
  return true;
}
// Thread 0 waits, the compute warps agree on the result.
DFSSM_DEV bool mbar_wait_compute(unsigned* status, unsigned* ctl, uint64_t* bar, unsigned parity, unsigned bit) {
  bool ok = true;
  if (threadIdx.x == 0) ok = mbar_wait(status, ctl, bar, parity, bit);
  return csync_and(ok);
}
// Cluster exchange: thread 0 arms the barrier with the bytes the cluster sends to
// this CTA (the sends may already have landed: the transaction count may run ahead
// of the arm) and waits (bounded) for the phase, the compute warps agree, then every
// thread takes the phase once more to acquire the cluster's writes for itself.
DFSSM_DEV bool xwait(unsigned* status, unsigned* ctl, uint64_t* bar, unsigned bytes, unsigned parity, unsigned bit) {
  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_expect_tx(bar, bytes);
    long long spins = 0;
    while (!mbar_try_wait_cluster(bar, parity)) {
      if (((++spins & 255) == 0) && (spins > spin_limit(ctl) || aborted(ctl))) {
        give_up(status, ctl, bit);
        ok = false;
        break;
      }
    }
  }
  ok = csync_and(ok);
  if (ok) (void)mbar_try_wait_cluster(bar, parity);
  return ok;
}

// Compute-warp reductions (fixed order, identical in every CTA).
DFSSM_DEV double csum_d(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_d(v);
  if (lane == 0) red[warp] = v;
  csync();
  double t = lane < kPWarps ? red[lane] : 0.0;
  t = warp_sum_d(t);
  csync();
  return t;
}
// Sum of the fp64 partials published by the grid's CTAs (word pairs), by every warp
// for itself (a fixed butterfly: every lane of every warp gets the same value).
DFSSM_DEV double sum_partials(const uint32_t* words, int G) {
  const int lane = threadIdx.x & 31;
  double t = 0.0;
  for (int c = lane; c < G; c += 32) t += f64_of(words + 2 * c);
  return warp_sum_d(t);
}
DFSSM_DEV long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------------ assignment

struct PWork {
  int c, k, r;           // CTA, cluster, rank inside the cluster
  int u0, nu;            // SSM units [u0, u0 + nu)
  int h0, h1;            // heads of those units
  int nbc;               // B/C tiles (2N/16)
  int cdt0, NS;          // the cluster's first dt tile (relative to dt_tile0), its shared tile count
  int s0, ns;            // own shared tiles [s0, s0 + ns) (B/C tiles first, then dt tiles)
  int nsbc;              // own shared tiles that are B/C tiles
  int ntile;             // in_proj tiles: nu z tiles, nu x tiles, ns shared tiles
  int o0, no;            // own out_proj tiles
};

// The same function runs on the host when the launch is planned.
__host__ __device__ inline PWork assign_cta(int c, int G, int Q, int units, int P, int n_bc_tiles, int out_tiles) {
  PWork w;
  w.c = c;
  w.k = c / Q;
  w.r = c % Q;
  auto ubeg = [&](int i) { return int((long long)i * units / G); };
  w.u0 = ubeg(c);
  w.nu = ubeg(c + 1) - w.u0;
  w.h0 = (16 * w.u0) / P;
  w.h1 = w.nu > 0 ? (16 * (w.u0 + w.nu) - 1) / P : w.h0 - 1;
  const int cu0 = ubeg(w.k * Q), cu1 = ubeg(w.k * Q + Q);
  int cndt = 0;
  w.cdt0 = 0;
  if (cu1 > cu0) {
    const int hl = (16 * cu0) / P, hh = (16 * cu1 - 1) / P;
    w.cdt0 = hl / 16;
    cndt = hh / 16 - hl / 16 + 1;
  }
  w.nbc = n_bc_tiles;
  w.NS = w.nbc + cndt;
  // Shared tiles even out the in_proj tiles (2 per unit + shared) over the ranks:
  // rank rr's share of the cluster's total, less its own z and x tiles; the last
  // rank takes what is left.
  const int T = 2 * (cu1 - cu0) + w.NS;
  int acc = 0;
  w.s0 = 0;
  w.ns = 0;
  for (int rr = 0; rr < Q; ++rr) {
    const int c2 = w.k * Q + rr;
    const int nu_rr = ubeg(c2 + 1) - ubeg(c2);
    const int t_rr = (rr + 1) * T / Q - rr * T / Q;
    int ns_rr = t_rr - 2 * nu_rr;
    ns_rr = ns_rr < 0 ? 0 : (ns_rr > w.NS - acc ? w.NS - acc : ns_rr);
    if (rr == Q - 1) ns_rr = w.NS - acc;
    if (rr == w.r) {
      w.s0 = acc;
      w.ns = ns_rr;
    }
    acc += ns_rr;
  }
  const int e = w.s0 + w.ns < w.nbc ? w.s0 + w.ns : w.nbc;
  w.nsbc = e > w.s0 ? e - w.s0 : 0;
  w.ntile = 2 * w.nu + w.ns;
  // out_proj tiles in reverse CTA order: the CTAs that hold an extra SSM unit (the
  // last of every run of the unit split) then never also hold an extra out tile
  const int rc = G - 1 - c;
  w.o0 = int((long long)rc * out_tiles / G);
  w.no = int((long long)(rc + 1) * out_tiles / G) - w.o0;
  return w;
}

DFSSM_DEV PWork assign(const PParams& a) {
  return assign_cta(int(blockIdx.x), a.grid, a.Q, a.units, a.P, a.n_bc_tiles, a.out_tiles);
}

// The four contiguous tile ranges of a CTA's in_proj rows: (first tile, count).
DFSSM_DEV void tile_range(const PParams& a, const PWork& w, int k, int* t0, int* n) {
  switch (k) {
    case 0: *t0 = w.u0; *n = w.nu; break;                                     // z rows
    case 1: *t0 = a.E / 16 + w.u0; *n = w.nu; break;                          // x rows
    case 2: *t0 = 2 * a.E / 16 + w.s0; *n = w.nsbc; break;                    // own B/C tiles
    default: {                                                                // own dt tiles
      const int b = max(w.s0, w.nbc);
      *t0 = a.dt_tile0 + w.cdt0 + (b - w.nbc);
      *n = w.ns - w.nsbc;
      break;
    }
  }
}

// in_proj tile index of tile slot ti (slots ordered z, x, B/C, dt)
DFSSM_DEV int slot_tile(const PParams& a, const PWork& w, int ti) {
  int t0, n;
  for (int k = 0; k < 4; ++k) {
    tile_range(a, w, k, &t0, &n);
    if (ti < n) return t0 + ti;
    ti -= n;
  }
  return -1;
}

template <typename T>
DFSSM_DEV T* sp(unsigned char* sm, int off) { return reinterpret_cast<T*>(sm + off); }

// ------------------------------------------------------------------ producer

// The issuing warp's copies are all bulk copies (the TMA engine moves the bytes; no
// per-16-byte requests that would stall the warp), spread over its 32 lanes: the
// k-th copy of a group is issued by lane k % 32.  Every copy completes on the
// group's mbarrier; lane 0 arms it with the group's total bytes (count pass first).
struct CopyList {
  unsigned char* sm;
  uint64_t* bar;
  int lane, k;
  bool issue;
  unsigned bytes;
  DFSSM_DEV void put(int dst_off, const void* src, int n) {
    if (n <= 0) return;
    if (issue) {
      if ((k & 31) == lane) bulk_g2s(sm + dst_off, src, unsigned(n), bar);
      ++k;
    } else {
      bytes += unsigned(n);
    }
  }
  // rows [0, rows) of `width` bytes, source row stride `stride`, into consecutive rows
  DFSSM_DEV void rows(int dst_off, const unsigned char* src, int rows, int width, size_t stride) {
    for (int j = 0; j < rows; ++j) put(dst_off + j * width, src + size_t(j) * stride, width);
  }
};

template <class F>
DFSSM_DEV void issue_group(unsigned char* sm, uint64_t* bar, F&& list) {
  const int lane = threadIdx.x & 31;
  CopyList c{sm, bar, lane, 0, false, 0u};
  list(c);
  if (lane == 0) mbar_expect_tx(bar, c.bytes);
  __syncwarp();
  c.issue = true;
  list(c);
}

// The AB group of layer l: this CTA's in_proj tiles, their LoRA B rows and scales,
// its slice of every LoRA A row, the whole pre-norm weight, its SSM state rows and
// the conv weights and state of its x channels and B/C rows.
DFSSM_BIG void produce_ab(const PParams& a, const PWork& w, const PLayer& L, unsigned char* sm, uint64_t* full) {
  const PSmem& s = a.sm;
  issue_group(sm, full, [&](CopyList& c) {
    const int tile_bytes = a.kg_in * 512;
    int slot = 0;
    for (int k = 0; k < 4; ++k) {
      int t0, n;
      tile_range(a, w, k, &t0, &n);
      if (n <= 0) continue;
      c.put(s.in_tiles + slot * tile_bytes, L.in_bits + size_t(t0) * a.kg_in * 128, n * tile_bytes);
      if (a.R) c.put(s.in_bq + slot * 16 * a.R, L.in_B + size_t(t0) * 16 * a.R, n * 16 * a.R);
      c.put(s.in_alpha + slot * 32, L.in_alpha + size_t(t0) * 16, n * 32);
      c.put(s.in_sb + slot * 32, (L.in_sB ? L.in_sB : L.in_alpha) + size_t(t0) * 16, n * 32);
      slot += n;
    }
    c.put(s.prenorm, L.prenorm_w, 2 * a.D);
    c.put(s.state, L.ssm_state + size_t(16 * w.u0) * a.N, w.nu * 16 * a.N * 4);
    const int ch = 16 * w.u0;
    c.put(s.convw_x, L.conv_w + size_t(ch) * 4, w.nu * 128);
    c.put(s.convb_x, L.conv_b + ch, w.nu * 32);
    for (int r = 0; r < 3; ++r) c.put(s.cst_x + r * kPMaxUnits * 64, L.conv_state + size_t(r) * a.C + ch, w.nu * 64);
    const int bch = a.E + 16 * w.s0;               // conv channel of the first own B/C row
    c.put(s.sh_convw, L.conv_w + size_t(bch) * 4, w.nsbc * 128);
    c.put(s.sh_convb, L.conv_b + bch, w.nsbc * 32);
    for (int r = 0; r < 3; ++r) c.put(s.sh_cst + r * kPMaxShared * 64, L.conv_state + size_t(r) * a.C + bch, w.nsbc * 64);
    if (a.R) {
      c.rows(s.a_in, reinterpret_cast<const unsigned char*>(L.in_A) + size_t(w.r) * a.SD, a.R, a.SD, size_t(a.D));
      c.put(s.sa_in, L.in_sA, 2 * a.R);
    }
    c.put(s.hd_dtb, L.dt_bias, 4 * a.H);
    c.put(s.hd_alog, L.A_log, 4 * a.H);
    c.put(s.hd_d, L.D, 4 * a.H);
  });
}

// The CD group of layer l: this CTA's out_proj tiles with their LoRA B rows and
// scales, its slice of every LoRA A row and the whole gated-norm weight.
DFSSM_BIG void produce_cd(const PParams& a, const PWork& w, const PLayer& L, unsigned char* sm, uint64_t* full) {
  const PSmem& s = a.sm;
  issue_group(sm, full, [&](CopyList& c) {
    const int tile_bytes = a.kg_out * 512;
    c.put(s.gnorm, L.gnorm_w, 2 * a.E);
    c.put(s.out_tiles, L.out_bits + size_t(w.o0) * a.kg_out * 128, w.no * tile_bytes);
    if (a.R) {
      c.put(s.out_bq, L.out_B + size_t(w.o0) * 16 * a.R, w.no * 16 * a.R);
      c.rows(s.a_out, reinterpret_cast<const unsigned char*>(L.out_A) + size_t(w.r) * a.SE, a.R, a.SE, size_t(a.E));
      c.put(s.sa_out, L.out_sA, 2 * a.R);
    }
    c.put(s.out_alpha, L.out_alpha + size_t(w.o0) * 16, w.no * 32);
    c.put(s.out_sb, (L.out_sB ? L.out_sB : L.out_alpha) + size_t(w.o0) * 16, w.no * 32);
  });
}

// ------------------------------------------------------------------ activation prep

// fp16 bits of z = (v * rs) * w correctly rounded from the fp64 product: the fp32
// product lies within 4 fp32 ulps of it, so when its low 13 mantissa bits are more
// than 4 away from the fp16 rounding midpoint (0x1000) and z is in the fp16 normal
// range, the hardware fp32 -> fp16 rounding of it is already the answer; otherwise
// fp64 decides.
DFSSM_DEV uint32_t norm_half(float v, double rs, float rs32, float wf) {
  const float z = (v * rs32) * wf;
  const float az = fabsf(z);
  const int low13 = int(__float_as_uint(z) & 0x1fffu);
  if (az >= 6.103515625e-05f && az < 65504.f && abs(low13 - 0x1000) > 4) return __half_as_ushort(__float2half_rn(z));
  return d2h((double(v) * rs) * double(wf));
}

// X = x 2^24 of one fp16 value as balanced base-256 digits (planes 0-3 in lo, 4-5 in
// the low bytes of hi), and its contribution to the exact sum split as X = xh 2^20 + xl.
// For |x| <= 127 (the usual case) X fits int32 and the four digits come from one add
// and one xor; larger values take the 64-bit path.
DFSSM_DEV void digits_and_sum(uint32_t h, uint32_t* lo, uint32_t* hi, int* xh, int* xl) {
  const uint32_t ha = h & 0x7fffu;
  if (ha <= 0x57f0u) {
    const uint32_t e = ha >> 10, m = ha & 0x3ffu;
    int X = e ? int((m | 0x400u) << (e - 1u)) : int(m);
    X = (h & 0x8000u) ? -X : X;
    *lo = (uint32_t(X) + 0x80808080u) ^ 0x80808080u;
    *hi = 0u;
    *xh += X >> 20;
    *xl += X & 0xfffff;
    return;
  }
  digits_of(h, lo, hi);
  const long long X = half_times_2p24_64(h);
  *xh += int(X >> 20);
  *xl += int(X & 0xfffff);
}

// Whole-vector preparation by the compute threads: x = fp16((v rs) w) for all K
// columns, their six digit planes (plane stride PS), the fp16 bits of the LoRA slice
// [s0, s0 + S) into xs, and -- identical in every thread -- the exact sum of X = x 2^24
// and max |x| (fp16 bits).  Four consecutive columns per thread and pass: the four
// digit words are transposed into one word per plane with eight byte permutes.
// `red` holds 3 ints per warp; it is read after the block barrier here, so the
// caller puts a barrier before its next use.
DFSSM_BIG void prep_full(const float* v, const uint16_t* w, int K, double rs, unsigned char* planes, int PS, int s0,
                         int S, uint16_t* xs, int* red, long long* xsum, unsigned* amax, uint16_t* x_diag,
                         int8_t* xd_diag) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float rs32 = float(rs);
  int xh = 0, xl = 0;
  unsigned am = 0;
  const int PW = PS / 4;
  for (int g = tid; g < K / 4; g += kPThreads) {
    const float4 v4 = reinterpret_cast<const float4*>(v)[g];
    const uint2 w4 = reinterpret_cast<const uint2*>(w)[g];
    const float2 wa = __half22float2(*reinterpret_cast<const __half2*>(&w4.x));
    const float2 wb = __half22float2(*reinterpret_cast<const __half2*>(&w4.y));
    const uint32_t h0 = norm_half(v4.x, rs, rs32, wa.x), h1 = norm_half(v4.y, rs, rs32, wa.y);
    const uint32_t h2 = norm_half(v4.z, rs, rs32, wb.x), h3 = norm_half(v4.w, rs, rs32, wb.y);
    uint32_t l0, l1, l2, l3, i0, i1, i2, i3;
    digits_and_sum(h0, &l0, &i0, &xh, &xl);
    digits_and_sum(h1, &l1, &i1, &xh, &xl);
    digits_and_sum(h2, &l2, &i2, &xh, &xl);
    digits_and_sum(h3, &l3, &i3, &xh, &xl);
    am = max(max(am, max(h0 & 0x7fffu, h1 & 0x7fffu)), max(h2 & 0x7fffu, h3 & 0x7fffu));
    // 4 x 4 byte transpose: plane d gets byte d of each column's digit word
    const uint32_t t0 = __byte_perm(l0, l1, 0x5140), t1 = __byte_perm(l0, l1, 0x7362);
    const uint32_t t2 = __byte_perm(l2, l3, 0x5140), t3 = __byte_perm(l2, l3, 0x7362);
    uint32_t* pw = reinterpret_cast<uint32_t*>(planes) + g;
    const uint32_t p0 = __byte_perm(t0, t2, 0x5410), p1 = __byte_perm(t0, t2, 0x7632);
    const uint32_t p2 = __byte_perm(t1, t3, 0x5410), p3 = __byte_perm(t1, t3, 0x7632);
    uint32_t p4 = 0u, p5 = 0u;
    if ((i0 | i1 | i2 | i3) != 0u) {
      p4 = __byte_perm(__byte_perm(i0, i1, 0x0040), __byte_perm(i2, i3, 0x0040), 0x5410);
      p5 = __byte_perm(__byte_perm(i0, i1, 0x0051), __byte_perm(i2, i3, 0x0051), 0x5410);
    }
    pw[0] = p0;
    pw[PW] = p1;
    pw[2 * PW] = p2;
    pw[3 * PW] = p3;
    pw[4 * PW] = p4;
    pw[5 * PW] = p5;
    const uint2 hh = make_uint2(h0 | (h1 << 16), h2 | (h3 << 16));
    const int c0 = 4 * g - s0;
    if (c0 >= 0 && c0 < S) *reinterpret_cast<uint2*>(xs + c0) = hh;
    if (x_diag) {
      *reinterpret_cast<uint2*>(x_diag + 4 * g) = hh;
      const uint32_t pp[6] = {p0, p1, p2, p3, p4, p5};
#pragma unroll
      for (int d = 0; d < kDigits; ++d) *reinterpret_cast<uint32_t*>(xd_diag + size_t(d) * K + 4 * g) = pp[d];
    }
  }
  // per thread |xh|, xl < 2^24: 32-lane sums fit int32; the warps' sums are combined in int64
  const int sh = __reduce_add_sync(0xffffffffu, xh);
  const int sl = __reduce_add_sync(0xffffffffu, xl);
  const unsigned amw = __reduce_max_sync(0xffffffffu, am);
  if (lane == 0) {
    red[3 * warp] = sh;
    red[3 * warp + 1] = sl;
    red[3 * warp + 2] = int(amw);
  }
  csync();
  long long s = 0;
  unsigned m = 0;
  if (lane < kPWarps) {
    s = (static_cast<long long>(red[3 * lane]) << 20) + red[3 * lane + 1];
    m = unsigned(red[3 * lane + 2]);
  }
  *xsum = warp_sum_ll(s);
  *amax = __reduce_max_sync(0xffffffffu, m);
}

// Digit-plane sums of the whole vector (diagnostics only), by all compute threads.
DFSSM_BIG void plane_sums(const unsigned char* planes, int PS, int K, int* red, int* out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int d = 0; d < kDigits; ++d) {
    int t = 0;
    for (int i = tid; i < K; i += kPThreads) t += int(int8_t(planes[d * PS + i]));
    t = __reduce_add_sync(0xffffffffu, t);
    if (lane == 0) red[warp] = t;
    csync();
    if (tid == 0) {
      int v = 0;
      for (int w = 0; w < kPWarps; ++w) v += red[w];
      out[d] = v;
    }
    csync();
  }
}

// int8 codes of the LoRA slice (from its fp16 bits), then the slice's LoRA stage-1
// partials of all R rows, sum_k A[j][k] q[k], sent by st.async to slot r of every
// CTA of the cluster (Q x R int32 land on each CTA's barrier `bar`).
DFSSM_BIG void codes_and_lora_send(const uint16_t* xs, int S, float sx, float rcp, bool nonzero, int8_t* xqs,
                                   const int8_t* Aslice, int R, int r, int Q, int* rcv, uint64_t* bar,
                                   int8_t* xq_diag) {
  const int tid = threadIdx.x;
  for (int i = tid; i < S; i += kPThreads) {
    const int q = nonzero ? quant_code_bits(half_to_float_bits(xs[i]), sx, rcp) : 0;
    xqs[i] = int8_t(q);
    if (xq_diag) xq_diag[i] = int8_t(q);
  }
  csync();
  if (R > 0) {
    // 16 lanes per row, two rows per warp; rows beyond the first pass of the warps
    // come round again (R is even, so both halves of a warp run the same passes)
    const int half = (tid & 31) >> 4, sub = tid & 15;
    const uint32_t dst0 = smem_u32(rcv + r * R), bar0 = smem_u32(bar);
    for (int j = 2 * (tid >> 5) + half; j < R; j += 2 * kPWarps) {
      const int* A4 = reinterpret_cast<const int*>(Aslice + j * S);
      const int* q4 = reinterpret_cast<const int*>(xqs);
      int acc = 0;
      for (int i = sub; i < S / 4; i += 16) acc = __dp4a(A4[i], q4[i], acc);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      // lanes 0..Q-1 of the half-warp each send the row's partial to one CTA
      if (sub < Q) st_async_b32(cluster_map(dst0 + 4 * j, sub), uint32_t(acc), cluster_map(bar0, sub));
    }
  }
}

// Sum of the cluster's LoRA partials (fixed order) -> u[j] = acc sA[j] sx in fp64.
DFSSM_BIG void lora_finish(const int* rcv, int Q, int R, const uint16_t* sA, float sx, double* u, int* acc_diag,
                           double* u_diag) {
  const int j = threadIdx.x;
  if (j < R) {
    int acc = 0;
    for (int q = 0; q < Q; ++q) acc += rcv[q * R + j];
    const double uj = (double(acc) * h2d(sA[j])) * double(sx);
    u[j] = uj;
    if (acc_diag) {
      acc_diag[j] = acc;
      u_diag[j] = uj;
    }
  }
  csync();
}

// Exact scaffold MMA over `ntile` tiles (smem, kg groups each), split into units
// (tile, kgroup chunk); int32 partials to part[unit][16][kDigits].  The activation
// digit planes are whole-vector planes (stride PS).  Register q of the A fragment of
// product s is word q of the lane's sign vector masked to bits s, s + 8, s + 16,
// s + 24: unsigned bytes 0 or 2^s, one instruction per register.  Product s
// accumulates into its own set, 2^s times its 0/1 sums (|sum| < 2^27), and the sets
// are recombined exactly with right shifts.  One 16-byte load per plane row gives
// the B fragments of products 2m and 2m + 1; the next k-group's words and planes are
// loaded while the current one's products issue.  Returns the chunks per tile.
DFSSM_BIG int scaffold_mma(const unsigned char* tiles, int ntile, int kg, const unsigned char* planes, int PS,
                           int* part) {
  constexpr int nw = kPWarps;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  int nchunk = nw / max(ntile, 1);
  if (nchunk < 1) nchunk = 1;
  if (nchunk > kg) nchunk = kg;
  const int nunits = ntile * nchunk;
  const unsigned char* dbase = planes + (g < kDigits ? g : 0) * PS + 16 * t;
  for (int unit = warp; unit < nunits; unit += nw) {
    const int ti = unit / nchunk, ci = unit % nchunk;
    const int kg_lo = ci * kg / nchunk, kg_hi = (ci + 1) * kg / nchunk;
    int acc[8][4];
#pragma unroll
    for (int s = 0; s < 8; ++s) acc[s][0] = acc[s][1] = acc[s][2] = acc[s][3] = 0;
    const uint4* tw = reinterpret_cast<const uint4*>(tiles + size_t(ti) * kg * 512);
    uint4 wv = tw[kg_lo * 32 + lane];
    uint4 bq[4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
      bq[m] = g < kDigits ? *reinterpret_cast<const uint4*>(dbase + kg_lo * kTileCols + 64 * m) : make_uint4(0, 0, 0, 0);
    for (int kgi = kg_lo; kgi < kg_hi; ++kgi) {
      uint4 wn = wv, bn[4] = {bq[0], bq[1], bq[2], bq[3]};
      if (kgi + 1 < kg_hi) {
        wn = tw[(kgi + 1) * 32 + lane];
#pragma unroll
        for (int m = 0; m < 4; ++m)
          if (g < kDigits) bn[m] = *reinterpret_cast<const uint4*>(dbase + (kgi + 1) * kTileCols + 64 * m);
      }
      const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t mask = 0x01010101u << (2 * m + e);
          const uint32_t af[4] = {words[0] & mask, words[1] & mask, words[2] & mask, words[3] & mask};
          mma_u8s8_16832(acc[2 * m + e], af, e ? bq[m].z : bq[m].x, e ? bq[m].w : bq[m].y);
        }
      }
      wv = wn;
#pragma unroll
      for (int m = 0; m < 4; ++m) bq[m] = bn[m];
    }
    int tot[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      tot[i] = acc[0][i];
#pragma unroll
      for (int s = 1; s < 8; ++s) tot[i] += acc[s][i] >> s;   // exact: acc[s] is a multiple of 2^s
    }
    int* pp = part + unit * 16 * kDigits;
    if (2 * t < kDigits) {
      pp[g * kDigits + 2 * t] = tot[0];
      pp[(g + 8) * kDigits + 2 * t] = tot[2];
    }
    if (2 * t + 1 < kDigits) {
      pp[g * kDigits + 2 * t + 1] = tot[1];
      pp[(g + 8) * kDigits + 2 * t + 1] = tot[3];
    }
  }
  csync();
  return nchunk;
}

// The unit partials of `ntile` tiles summed over their chunks into a [ntile][16][6]
// table, one compute thread per (tile, row, digit), in chunk order.
DFSSM_DEV void combine_parts(const int* part, int ntile, int nchunk, int* tbl) {
  for (int i = threadIdx.x; i < ntile * 16 * kDigits; i += kPThreads) {
    const int ti = i / (16 * kDigits), rd = i % (16 * kDigits);
    int s = 0;
    for (int c = 0; c < nchunk; ++c) s += part[(ti * nchunk + c) * 16 * kDigits + rd];
    tbl[i] = s;
  }
  csync();
}
// Scaffold value (without alpha) of table row i: 2^-24 (2 sum_d 256^d Q_d - sum_k X_k).
DFSSM_DEV double table_row_value(const int* tbl, int i, long long xsum) {
  long long S = 0;
#pragma unroll
  for (int d = kDigits - 1; d >= 0; --d) S = S * 256 + tbl[i * kDigits + d];
  return double(2 * S - xsum) * (1.0 / 16777216.0);
}
// LoRA stage 2 of `nrows` rows, out[r] = sum_j B[r][j] u[j] in fp64, four lanes per row
// (lane q takes the terms j = q mod 4), combined as (q0 + q1) + (q2 + q3).
DFSSM_DEV void lora2_all(const int8_t* Bq, int nrows, const double* u, int R, double* out) {
  const int q = threadIdx.x & 3;
  for (int base = 0; base < nrows * 4; base += kPThreads) {
    const int i = base + int(threadIdx.x), r = i >> 2;
    double acc = 0.0;
    if (r < nrows) {
      const int8_t* br = Bq + r * R;
      for (int j = q; j < R; j += 4) acc = fma(double(br[j]), u[j], acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (q == 0 && r < nrows) out[r] = acc;
  }
  csync();
}

// Pre-activation of one conv channel: bias + taps 0..2 on the stored inputs (oldest
// first) + tap 3 on the new input, in fp64.
DFSSM_DEV double conv_step_d(const uint16_t* cw, double cb, float c0, float c1, float c2, double xv) {
  double pre = cb;
  pre = fma(h2d(cw[0]), double(c0), pre);
  pre = fma(h2d(cw[1]), double(c1), pre);
  pre = fma(h2d(cw[2]), double(c2), pre);
  pre = fma(h2d(cw[3]), xv, pre);
  return pre;
}

// ------------------------------------------------------------------ the kernel

template <class SH, bool Q8>
__global__ void __launch_bounds__(kPBlock, 1) k_decode_persistent(const __grid_constant__ PParams pa) {
  extern __shared__ __align__(128) unsigned char sm[];
  // The parameter block (~11 KB, mostly the per-layer pointer table) is read with
  // runtime layer indices all through the token; a shared-memory copy keeps those
  // reads off the small constant cache.
  __shared__ __align__(16) unsigned char pbuf[sizeof(PParams)];
  __shared__ __align__(8) uint64_t bars[4 + 2 * kHeadRingMax];   // full/empty AB, CD and head slots
  __shared__ __align__(8) uint64_t xbars[EX_N];
  __shared__ double redd[kPWarps];
  __shared__ int redi[3 * kPWarps];
  __shared__ int redo[3 * kPWarps];
  __shared__ double ssw[kPWarps * kPSsmRows];
  __shared__ int s_stale, s_withhold;
  for (int i = threadIdx.x; i < int(sizeof(PParams) / 16); i += blockDim.x)
    reinterpret_cast<uint4*>(pbuf)[i] = reinterpret_cast<const uint4*>(&pa)[i];
  const PParams& a = *reinterpret_cast<const PParams*>(pbuf);
  const PWork w = assign(pa);
  // sizes: compile-time for a fixed shape, else from the parameters
  constexpr bool kC = SH::kConst;
  const int D = kC ? SH::D : pa.D, E = kC ? SH::E : pa.E, P = kC ? SH::P : pa.P, N = kC ? SH::N : pa.N;
  const int R = kC ? SH::R : pa.R, C = kC ? SH::C : pa.C, Q = kC ? SH::Q : pa.Q;
  const int kg_in = kC ? SH::kg_in : pa.kg_in, kg_out = kC ? SH::kg_out : pa.kg_out;
  const int SD = kC ? SH::SD : pa.SD, SE = kC ? SH::SE : pa.SE;
#define PSM(f) (kC ? SH::kPlan.f : pa.sm.f)
  uint64_t* full_ab = &bars[0];
  uint64_t* empty_ab = &bars[1];
  uint64_t* full_cd = &bars[2];
  uint64_t* empty_cd = &bars[3];
  uint64_t* full_h = &bars[4];
  uint64_t* empty_h = &bars[4 + kHeadRingMax];
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4 + kHeadRingMax; ++i) mbar_init(&bars[i], 1);
    for (int i = 0; i < kHeadRingMax; ++i) mbar_init(&bars[4 + kHeadRingMax + i], kPWarps);   // head slots: one arrival per compute warp
    for (int i = 0; i < EX_N; ++i) mbar_init(&xbars[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // An abort flag left by an earlier call means its exchange words may still carry
    // this launch's epoch: do nothing and say so (the caller zero-fills the workspace).
    s_stale = aborted(pa.ctl) ? 1 : 0;
    if (s_stale) atomicOr(pa.status, 1u);
    s_withhold = int(*reinterpret_cast<volatile const unsigned*>(pa.ctl + 2));
  }
  // every CTA's barriers exist before any CTA of the cluster copies into it
  cluster_sync_all();
  const bool stale = s_stale != 0;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.grid;
  const int v0 = int((long long)w.c * a.vocab / G), v1 = int((long long)(w.c + 1) * a.vocab / G);
  // LM-head rows: fp16, or (Q8) int8 codes with a per-row scale.  Slots are spaced for
  // 15 fp16 rows, which is 30 int8 rows: an int8 chunk is 30 rows (half the chunks).
  // A compile-time choice keeps the fp16 kernel's registers as they were.
  constexpr bool q8 = Q8;
  constexpr int CR = Q8 ? 2 * kHeadChunkRows : kHeadChunkRows;
  const unsigned head_row_bytes = q8 ? unsigned(D) : 2u * D;
  const int head_chunks = (v1 - v0 + CR - 1) / CR;

  // LM-head chunk slots tile the shared memory below `ring_end`; the slots inside
  // the AB group are free after the last layer's SSM, the others after its out_proj
  const int NH = PSM(head_slots);
  const int chunk_bytes = kHeadChunkRows * 2 * D;
  auto head_slot = [&](int b) { return sm + b * chunk_bytes; };
  if (stale) {
    // nothing issued, nothing to wait for
  } else if (warp == kPWarps) {
    // ============================================================== copy warp
    bool ok = true;
    unsigned ab_issued = 0, cd_issued = 0, h_issued[kHeadRingMax] = {};
    auto wait = [&](uint64_t* bar, unsigned parity, unsigned bit) {
      if (lane == 0) ok = mbar_wait(a.status, a.ctl, bar, parity, bit);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      return ok;
    };
    auto issue_head = [&](int ci) {
      const int b = ci % NH;
      const int r0 = v0 + ci * CR, nr = min(CR, v1 - r0);
      if (lane == 0) {
        mbar_expect_tx(full_h + b, nr * head_row_bytes);
        const void* src = q8 ? static_cast<const void*>(a.embed_q + size_t(r0) * D)
                             : static_cast<const void*>(a.embed + size_t(r0) * D);
        bulk_g2s(head_slot(b), src, nr * head_row_bytes, full_h + b);
      }
      ++h_issued[b];
    };
    for (int l = 0; l < a.n_layer && ok; ++l) {
      if (l > 0 && !wait(empty_ab, unsigned(l - 1) & 1u, 4096u)) break;
      produce_ab(a, w, a.L[l], sm, full_ab);
      ++ab_issued;
      if (l > 0 && !wait(empty_cd, unsigned(l - 1) & 1u, 8192u)) break;
      produce_cd(a, w, a.L[l], sm, full_cd);
      ++cd_issued;
    }
    if (ok && !a.layer_mode) {
      const unsigned lp = unsigned(a.n_layer - 1) & 1u;
      int ci = 0;
      if (wait(empty_ab, lp, 4096u))
        for (; ci < NH && ci < head_chunks && (ci + 1) * chunk_bytes <= PSM(ab_end); ++ci) issue_head(ci);
      if (ok && wait(empty_cd, lp, 8192u)) {
        for (; ci < head_chunks && ok; ++ci) {
          const int b = ci % NH;
          if (ci >= NH && !wait(empty_h + b, unsigned(ci / NH - 1) & 1u, 16384u)) break;
          issue_head(ci);
        }
      }
    }
    // let every issued copy land before leaving (the CTA's shared memory stays
    // alive until all its threads exit)
    if (lane == 0) {
      long long spins = 0;
      if (ab_issued) while (!mbar_try_wait(full_ab, (ab_issued - 1) & 1u) && ++spins < kSpinLimit) {}
      if (cd_issued) while (!mbar_try_wait(full_cd, (cd_issued - 1) & 1u) && ++spins < kSpinLimit) {}
      for (int b = 0; b < kHeadRingMax; ++b)
        if (h_issued[b]) while (!mbar_try_wait(full_h + b, (h_issued[b] - 1) & 1u) && ++spins < kSpinLimit) {}
    }
    __syncwarp();
  } else {
    // ============================================================== compute warps
    const uint32_t tagbase = *reinterpret_cast<volatile const unsigned*>(a.ctl) << 16;   // launch epoch
    auto tag = [&](int l, int kind) { return tagbase + uint32_t(l * 8 + kind + 1); };
    unsigned* status = a.status;
    unsigned* ctl = a.ctl;
#ifdef DFSSM_PHASE_TIMERS
    long long ptime[PH_N];
#pragma unroll
    for (int i = 0; i < PH_N; ++i) ptime[i] = 0;
    long long tlast = clock64();
#define PT(k)                              \
  do {                                     \
    if (tid == 0) {                        \
      const long long t_ = clock64();      \
      ptime[k] += t_ - tlast;              \
      tlast = t_;                          \
    }                                      \
  } while (0)
#else
#define PT(k) \
  do {        \
  } while (0)
#endif

    float* vfull = sp<float>(sm, PSM(vfull));          // the whole residual / gated value
    unsigned char* planes = sm + PSM(planes);          // six digit planes of the activation
    uint16_t* xs = sp<uint16_t>(sm, PSM(xs));          // fp16 bits of this CTA's LoRA slice
    int8_t* xqs = sp<int8_t>(sm, PSM(xqs));
    int* rcv_in = sp<int>(sm, PSM(rcv));               // [Q][R] the cluster's in_proj LoRA partials
    int* rcv_out = rcv_in + Q * (R > 4 ? R : 4);       // [Q][R] the cluster's out_proj LoRA partials
    int* part = sp<int>(sm, PSM(part));
    double* yin = sp<double>(sm, PSM(yin));            // [kPMaxInTiles * 16] in_proj outputs of own tiles (slot order)
    double* shr = sp<double>(sm, PSM(shr));            // [kPMaxSharedRows] the cluster's shared rows
    float* shst = sp<float>(sm, PSM(shst));            // [3][kPMaxShared * 16] new conv state of own B/C rows
    double* u = sp<double>(sm, PSM(u));                // [R] LoRA stage-1 outputs
    float* resown = sp<float>(sm, PSM(resown));        // residual of own out_proj rows
    uint32_t* scratch32 = sp<uint32_t>(sm, PSM(full)); // gathered partial words, then the head's residual
    const int zslot = 0, xslot = w.nu, shslot = 2 * w.nu;
    const int SHR = kPMaxShared * 16;
    const int PSD = plane_stride(D), PSE = plane_stride(E);
    const int tile_in = kg_in * 512;
    const uint32_t shr_s = smem_u32(shr), xsh_s = smem_u32(&xbars[EX_SH]);
    // this CTA's shared rows start at cluster shared row 16 s0 + 16 (s0 - nbc)+
    const int shr_own = 16 * w.s0 + 16 * max(w.s0 - w.nbc, 0);

    // ---- layer-0 residual: the whole vector and its sum of squares (every CTA)
    double ss;
    {
      int t = 0;
      if (!a.layer_mode) {
        t = a.tok_in[0];
        if (t < 0 || t >= a.vocab) {
          if (tid == 0) atomicOr(status, 2u);
          t = t < 0 ? 0 : a.vocab - 1;
        }
      }
      const uint16_t* erow = a.embed + size_t(t) * D;
      const int8_t* eqrow = q8 ? a.embed_q + size_t(t) * D : nullptr;
      const float es = q8 ? a.embed_s[t] : 0.f;
      double acc = 0.0;
      for (int k = tid; k < D; k += kPThreads) {
        const float v = a.layer_mode ? a.residual[k] : q8 ? es * float(eqrow[k]) : h2f(erow[k]);
        vfull[k] = v;
        acc = fma(double(v), double(v), acc);
      }
      ss = csum_d(acc, redd);
      if (tid < w.no * 16) resown[tid] = vfull[w.o0 * 16 + tid];
    }

    bool alive = true;
    for (int l = 0; l < a.n_layer && alive; ++l) {
      const PLayer& L = a.L[l];
      const bool diag = (l == a.n_layer - 1);
      const bool cdiag = diag && w.k == 0;      // cluster 0 writes the slice diagnostics
      const bool wdiag = diag && w.c == 0;
      const unsigned par = unsigned(l) & 1u;

      // ---- R: the whole residual and the sums of squares
      if (l > 0) {
        if (!tw_gather<(2048 + 2 * 128 + kPThreads - 1) / kPThreads>(
                status, ctl, a.x_r, D, reinterpret_cast<uint32_t*>(vfull), a.x_rs, 2 * G, scratch32, tag(l, XR),
                4u)) {
          alive = false;
          break;
        }
        ss = sum_partials(scratch32, G);
      }
      PT(PH_GATHER_R);
      if (!mbar_wait_compute(status, ctl, full_ab, par, 8u)) { alive = false; break; }
      PT(PH_WAIT_AB);

      // ---- A: pre-norm of the whole vector, digit planes, sum, max
      const double rs_in = 1.0 / sqrt(ss / double(D) + kEpsD);
      long long xsum_in;
      unsigned amax_in;
      prep_full(vfull, sp<uint16_t>(sm, PSM(prenorm)), D, rs_in, planes, PSD, w.r * SD, SD, xs, redi, &xsum_in,
                &amax_in, wdiag ? a.d_x_in : nullptr, a.d_xd_in);
      const float am_in = half_to_float_bits(amax_in);
      const float sx_in = am_in > 0.f ? __fdiv_rn(am_in, 127.f) : 1.f;
      PT(PH_PREP_IN);
      // ---- L: codes and LoRA partials of the slice -> the cluster
      codes_and_lora_send(xs, SD, sx_in, __frcp_rn(sx_in), am_in > 0.f, xqs, sp<int8_t>(sm, PSM(a_in)), R, w.r, Q,
                          rcv_in, &xbars[EX_LIN], cdiag ? a.d_xq_in + w.r * SD : nullptr);
      if (wdiag) {
        if (tid == 0) *a.d_sx_in = sx_in;
        plane_sums(planes, PSD, D, redi, a.d_xdsum_in);
      }
      PT(PH_LORA_IN);
      // ---- S: the shared tiles (B/C rows, dt rows) first: the cluster waits for them
      int* tbl = sp<int>(sm, PSM(misc));                 // [tiles][16][6] chunk-summed digit sums
      double* lo = sp<double>(sm, PSM(lo2));            // LoRA stage-2 sums of own in_proj rows (slot order)
      int nch = 1;
      if (w.ns > 0) {
        nch = scaffold_mma(sm + PSM(in_tiles) + shslot * tile_in, w.ns, kg_in, planes, PSD, part);
        combine_parts(part, w.ns, nch, tbl);
      }
      if (tid < w.ns * 16)
        yin[shslot * 16 + tid] = h2d(sp<uint16_t>(sm, PSM(in_alpha))[shslot * 16 + tid]) * table_row_value(tbl, tid, xsum_in);
      PT(PH_MMA_SH);
      if (R) {
        if (!xwait(status, ctl, &xbars[EX_LIN], unsigned(Q * 4 * R), par, 16u)) { alive = false; break; }
        lora_finish(rcv_in, Q, R, sp<uint16_t>(sm, PSM(sa_in)), sx_in, u, wdiag ? a.d_acc_in : nullptr, a.d_u_in);
        // the shared rows first (the cluster waits for them); the z/x rows' after the send
        lora2_all(sp<int8_t>(sm, PSM(in_bq)) + shslot * 16 * R, w.ns * 16, u, R, lo + shslot * 16);
      }
      PT(PH_WAIT_LIN);
      // own shared rows: LoRA stage 2, then conv + SiLU (B/C) or step size + decay (dt),
      // each value sent to every CTA of the cluster.  Row i runs on thread
      // kPThreads - 1 - i: the last warps get no unit of the z/x scaffold MMA that
      // follows (fewer units than warps), so the step-size rows' fp64 softplus / exp
      // chain no longer delays a warp that holds one.
      if (kPThreads - 1 - tid < w.ns * 16) {
        const int i = kPThreads - 1 - tid;
        const int si = w.s0 + i / 16, r = i % 16;        // shared tile of the cluster, row in it
        double v = yin[shslot * 16 + i];
        if (R) v = fma(h2d(sp<uint16_t>(sm, PSM(in_sb))[shslot * 16 + i]), lo[shslot * 16 + i], v);
        if (diag) a.d_zx[slot_tile(a, w, shslot + i / 16) * 16 + r] = v;
        if (si < w.nbc) {                                 // a B/C row: conv step + SiLU
          const float* cst = sp<float>(sm, PSM(sh_cst));
          const float c0 = cst[i], c1 = cst[SHR + i], c2 = cst[2 * SHR + i];
          const double pre = conv_step_d(sp<uint16_t>(sm, PSM(sh_convw)) + i * 4,
                                         h2d(sp<uint16_t>(sm, PSM(sh_convb))[i]), c0, c1, c2, v);
          shst[i] = c1;
          shst[SHR + i] = c2;
          shst[2 * SHR + i] = float(v);
          const double xc = silu_d(pre);
          if (diag) a.d_xc[E + 16 * si + r] = xc;
          const unsigned long long bits = static_cast<unsigned long long>(__double_as_longlong(xc));
          for (int q = 0; q < Q; ++q)
            st_async_b64(cluster_map(shr_s + 8 * (shr_own + i), q), bits, cluster_map(xsh_s, q));
        } else {                                          // a dt row: step size and decay of its head
          const int h = 16 * (w.cdt0 + si - w.nbc) + r;
          const double dt = softplus_d(v + double(sp<float>(sm, PSM(hd_dtb))[h]));
          const double dA = exp(dt * -exp(double(sp<float>(sm, PSM(hd_alog))[h])));
          const int o = shr_own + 16 * w.nsbc + 32 * (i / 16 - w.nsbc) + r;   // dt tile: 16 steps, 16 decays
          const unsigned long long b0 = static_cast<unsigned long long>(__double_as_longlong(dt));
          const unsigned long long b1 = static_cast<unsigned long long>(__double_as_longlong(dA));
          for (int q = 0; q < Q; ++q) {
            st_async_b64(cluster_map(shr_s + 8 * o, q), b0, cluster_map(xsh_s, q));
            st_async_b64(cluster_map(shr_s + 8 * (o + 16), q), b1, cluster_map(xsh_s, q));
          }
        }
      }
      PT(PH_SHARED);
      // ---- Z: the z and x tiles of own SSM channels
      nch = scaffold_mma(sm + PSM(in_tiles), 2 * w.nu, kg_in, planes, PSD, part);
      combine_parts(part, 2 * w.nu, nch, tbl);
      if (R) lora2_all(sp<int8_t>(sm, PSM(in_bq)), 2 * w.nu * 16, u, R, lo);
      PT(PH_MMA_ZX);
      if (tid < 2 * w.nu * 16) {
        const int i = tid;
        double v = h2d(sp<uint16_t>(sm, PSM(in_alpha))[i]) * table_row_value(tbl, i, xsum_in);
        if (R) v = fma(h2d(sp<uint16_t>(sm, PSM(in_sb))[i]), lo[i], v);
        if (diag) a.d_zx[slot_tile(a, w, i / 16) * 16 + i % 16] = v;
        if (i < w.nu * 16) {                              // z row: the gate silu(z)
          yin[i] = silu_d(v);
        } else {                                          // x row: conv step + SiLU
          const int j = i - w.nu * 16;                    // channel within the CTA's units
          const int uu = j / 16, r = j % 16;
          const float* cst = sp<float>(sm, PSM(cst_x));
          const float c0 = cst[(0 * kPMaxUnits + uu) * 16 + r];
          const float c1 = cst[(1 * kPMaxUnits + uu) * 16 + r];
          const float c2 = cst[(2 * kPMaxUnits + uu) * 16 + r];
          const double pre = conv_step_d(sp<uint16_t>(sm, PSM(convw_x)) + j * 4,
                                         h2d(sp<uint16_t>(sm, PSM(convb_x))[j]), c0, c1, c2, v);
          const int ch = 16 * w.u0 + j;
          float* gcs = L.conv_state;
          gcs[ch] = c1;
          gcs[C + ch] = c2;
          gcs[2 * C + ch] = float(v);
          const double xc = silu_d(pre);
          yin[i] = xc;
          if (diag) a.d_xc[ch] = xc;
        }
      }
      PT(PH_ZX_EPI);
      if (!xwait(status, ctl, &xbars[EX_SH], unsigned((2 * w.NS - w.nbc) * 16 * 8), par, 32u)) {
        alive = false;
        break;
      }
      PT(PH_WAIT_SH);
      // ---- G: SSM update of own rows (warp per row, 4 states per lane per step);
      // publish g and the sum of its squares
      {
        const float* st = sp<float>(sm, PSM(state));
        const int nrow = w.nu * 16;
        double yv[kPSsmRows];
#pragma unroll
        for (int i = 0; i < kPSsmRows; ++i) {
          yv[i] = 0.0;
          const int rr = warp + kPWarps * i;
          if (rr < nrow) {
            const int e = 16 * w.u0 + rr;             // row of d_inner
            const int hh = e / P - 16 * w.cdt0;       // head within the cluster's dt tiles
            const double* dtt = shr + 2 * N + 32 * (hh / 16) + hh % 16;
            const double dA = dtt[16];
            const double xdt = yin[(xslot + rr / 16) * 16 + rr % 16] * dtt[0];
            const float4* hrow = reinterpret_cast<const float4*>(st + size_t(rr) * N);
            float4* grow = reinterpret_cast<float4*>(L.ssm_state + size_t(e) * N);
            const double2* B2 = reinterpret_cast<const double2*>(shr);
            const double2* C2 = reinterpret_cast<const double2*>(shr + N);
            double y = 0.0;
            for (int n4 = lane; n4 < N / 4; n4 += 32) {
              const float4 hv = hrow[n4];
              const double2 b01 = B2[2 * n4], b23 = B2[2 * n4 + 1];
              const double2 c01 = C2[2 * n4], c23 = C2[2 * n4 + 1];
              const double h0 = fma(dA, double(hv.x), xdt * b01.x);
              const double h1 = fma(dA, double(hv.y), xdt * b01.y);
              const double h2 = fma(dA, double(hv.z), xdt * b23.x);
              const double h3 = fma(dA, double(hv.w), xdt * b23.y);
              y = fma(c01.x, h0, y);
              y = fma(c01.y, h1, y);
              y = fma(c23.x, h2, y);
              y = fma(c23.y, h3, y);
              grow[n4] = make_float4(float(h0), float(h1), float(h2), float(h3));
            }
            yv[i] = y;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
          for (int i = 0; i < kPSsmRows; ++i) yv[i] += __shfl_xor_sync(0xffffffffu, yv[i], o);
        // lane i finishes row warp + kPWarps i: D skip, gate, publish g
        double g2 = 0.0;
#pragma unroll
        for (int i = 0; i < kPSsmRows; ++i) {
          const int rr = warp + kPWarps * i;
          if (lane == i && rr < nrow) {
            const int e = 16 * w.u0 + rr;
            const double x = yin[(xslot + rr / 16) * 16 + rr % 16];
            const double gate = yin[(zslot + rr / 16) * 16 + rr % 16];
            const double y = fma(double(sp<float>(sm, PSM(hd_d))[e / P]), x, yv[i]);
            const float gv = float(y * gate);
            tw_put(a.x_g + e, __float_as_uint(gv), tag(l, XG));
            if (diag) a.d_g[e] = gv;
            g2 = double(gv) * double(gv);
          }
        }
        if (lane < kPSsmRows) ssw[warp * kPSsmRows + lane] = g2;
      }
      csync();
      if (warp == 0) {          // sum of squares of the CTA's gated values (fixed order)
        double t = 0.0;
        for (int i = lane; i < kPWarps * kPSsmRows; i += 32) t += ssw[i];
        t = warp_sum_d(t);
        if (lane == 0) tw_put_f64(a.x_gs + 2 * w.c, t, tag(l, XG));
      }
      if (tid == 0) mbar_arrive(empty_ab);      // AB group consumed: the copy warp may refill it
      PT(PH_SSM);
      // ---- G: the whole gated value and the sums of squares
      if (!tw_gather<(4096 + 2 * 128 + kPThreads - 1) / kPThreads>(
              status, ctl, a.x_g, E, reinterpret_cast<uint32_t*>(vfull), a.x_gs, 2 * G, scratch32, tag(l, XG),
              64u)) {
        alive = false;
        break;
      }
      const double ssg = sum_partials(scratch32, G);
      if (w.k == 0) {   // B/C conv state of this layer: every CTA has finished reading it
        for (int i = tid; i < w.nsbc * 16; i += kPThreads) {
          const int ch = E + 16 * w.s0 + i;
          for (int r = 0; r < 3; ++r) L.conv_state[size_t(r) * C + ch] = shst[r * SHR + i];
        }
      }
      PT(PH_GATHER_G);
      if (!mbar_wait_compute(status, ctl, full_cd, par, 128u)) { alive = false; break; }
      PT(PH_WAIT_CD);
      // ---- A': gated RMSNorm of the whole vector
      const double rs_out = 1.0 / sqrt(ssg / double(E) + kEpsD);
      long long xsum_out;
      unsigned amax_out;
      prep_full(vfull, sp<uint16_t>(sm, PSM(gnorm)), E, rs_out, planes, PSE, w.r * SE, SE, xs, redo, &xsum_out,
                &amax_out, wdiag ? a.d_x_out : nullptr, a.d_xd_out);
      const float am_out = half_to_float_bits(amax_out);
      const float sx_out = am_out > 0.f ? __fdiv_rn(am_out, 127.f) : 1.f;
      PT(PH_PREP_OUT);
      // ---- L': codes and LoRA partials of the slice -> the cluster
      codes_and_lora_send(xs, SE, sx_out, __frcp_rn(sx_out), am_out > 0.f, xqs, sp<int8_t>(sm, PSM(a_out)), R,
                          w.r, Q, rcv_out, &xbars[EX_LOUT], cdiag ? a.d_xq_out + w.r * SE : nullptr);
      if (wdiag) {
        if (tid == 0) *a.d_sx_out = sx_out;
        plane_sums(planes, PSE, E, redo, a.d_xdsum_out);
      }
      PT(PH_LORA_OUT);
      // ---- O: out_proj scaffold on own tiles
      int* tbl_o = sp<int>(sm, PSM(misc));
      double* lo_o = sp<double>(sm, PSM(lo2));
      if (w.no > 0) {
        const int nch_out = scaffold_mma(sm + PSM(out_tiles), w.no, kg_out, planes, PSE, part);
        combine_parts(part, w.no, nch_out, tbl_o);
      }
      PT(PH_MMA_OUT);
      if (R) {
        if (!xwait(status, ctl, &xbars[EX_LOUT], unsigned(Q * 4 * R), par, 256u)) { alive = false; break; }
        lora_finish(rcv_out, Q, R, sp<uint16_t>(sm, PSM(sa_out)), sx_out, u, wdiag ? a.d_acc_out : nullptr,
                    a.d_u_out);
        lora2_all(sp<int8_t>(sm, PSM(out_bq)), w.no * 16, u, R, lo_o);
      }
      PT(PH_WAIT_LOUT);
      // ---- residual rows and their sum of squares, published for the next layer (a
      // test can make one CTA withhold its layer-0 words so that the next gather runs out)
      const bool last = (l + 1 == a.n_layer);
      const bool publish = !(last && a.layer_mode) && !(l == 0 && s_withhold == w.c + 1);
      if (tid < w.no * 16) {
        const int o = w.o0 * 16 + tid;
        double y = h2d(sp<uint16_t>(sm, PSM(out_alpha))[tid]) * table_row_value(tbl_o, tid, xsum_out);
        if (R) y = fma(h2d(sp<uint16_t>(sm, PSM(out_sb))[tid]), lo_o[tid], y);
        const float rn = float(double(resown[tid]) + y);
        resown[tid] = rn;
        if (publish) tw_put(a.x_r + o, __float_as_uint(rn), tag(l + 1, XR));
        if (last) {
          if (a.layer_mode) a.residual[o] = rn;
          else a.d_res[o] = rn;
        }
      }
      csync();
      if (warp == 0) {          // sum of squares of the CTA's residual rows (fixed order)
        double t = 0.0;
        for (int i = lane; i < w.no * 16; i += 32) t = fma(double(resown[i]), double(resown[i]), t);
        t = warp_sum_d(t);
        if (lane == 0 && publish) tw_put_f64(a.x_rs + 2 * w.c, t, tag(l + 1, XR));
      }
      if (tid == 0) mbar_arrive(empty_cd);      // CD group consumed
      PT(PH_RESID);
    }

    // ---- LM head
    if (alive && !a.layer_mode) {
      const int L = a.n_layer;
      // the final residual lands beyond the ring (the copy warp is already filling
      // chunk slots over the working buffers) and is normalised in place
      float* xn = reinterpret_cast<float*>(scratch32 + 2 * G);     // [D] residual, then normalised
      if (tw_gather<(2048 + 2 * 128 + kPThreads - 1) / kPThreads>(
              status, ctl, a.x_r, D, reinterpret_cast<uint32_t*>(xn), a.x_rs, 2 * G, scratch32, tag(L, XR),
              512u)) {
        const double rs = 1.0 / sqrt(sum_partials(scratch32, G) / double(D) + kEpsD);
        for (int k = tid; k < D; k += kPThreads) xn[k] = float((double(xn[k]) * rs) * h2d(a.normf_w[k]));
        csync();
        PT(PH_HEAD);
        // Every compute warp takes whole rows -- row `warp` of each 15-row group of a
        // chunk (one group per fp16 chunk, two per int8 chunk) -- waits on the chunk's
        // slot itself and releases it with its own arrival (the empty barriers count
        // one arrival per compute warp), so no block barrier runs per chunk.  A lane
        // keeps its kHV 8-column groups of the normalised residual in registers.
        constexpr int kHV = 8;
        const int hn = D / 8;                        // 8-column groups per row
        float xr[kHV][8];
#pragma unroll
        for (int m = 0; m < kHV; ++m)
#pragma unroll
          for (int e = 0; e < 8; ++e) xr[m][e] = lane + 32 * m < hn ? xn[(lane + 32 * m) * 8 + e] : 0.f;
        auto f16x8 = [](const uint4& wv, float (&f)[8]) {
          const __half2* wh = reinterpret_cast<const __half2*>(&wv);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 t2 = __half22float2(wh[i]);
            f[2 * i] = t2.x;
            f[2 * i + 1] = t2.y;
          }
        };
        float best = -INFINITY;
        int besti = 0x7fffffff;
        bool hok = true;
        // int8 rows: lane 0 loads its rows' scales one chunk ahead, so the load's
        // latency is not paid after every row's reduction
        constexpr int RW = CR / kPWarps;             // rows per warp and chunk
        float scn[RW];
        auto load_scales = [&](int ci2) {
          const int r02 = v0 + ci2 * CR, nr2 = min(CR, v1 - r02);
#pragma unroll
          for (int rsub = 0; rsub < RW; ++rsub) {
            const int row = warp + kPWarps * rsub;
            scn[rsub] = (q8 && lane == 0 && row < nr2) ? __ldg(a.embed_s + r02 + row) : 1.f;
          }
        };
        if (q8 && head_chunks > 0) load_scales(0);
        for (int ci = 0; ci < head_chunks; ++ci) {
          const int b = ci % NH;
          float sc[RW];
#pragma unroll
          for (int rsub = 0; rsub < RW; ++rsub) sc[rsub] = scn[rsub];
          if (q8 && ci + 1 < head_chunks) load_scales(ci + 1);
          {   // every lane takes the slot's phase (bounded; lane 0 flags a timeout)
            long long spins = 0;
            while (!mbar_try_wait(full_h + b, unsigned(ci / NH) & 1u)) {
              if (((++spins & 255) == 0) && (spins > spin_limit(ctl) || aborted(ctl))) {
                if (lane == 0) give_up(status, ctl, 1024u);
                hok = false;
                break;
              }
            }
            hok = __all_sync(0xffffffffu, hok);
          }
          if (!hok) break;
          const int r0 = v0 + ci * CR, nr = min(CR, v1 - r0);
#pragma unroll
          for (int rsub = 0; rsub < RW; ++rsub) {
            const int row = warp + kPWarps * rsub;
            if (row < nr) {
              const unsigned char* wrow = head_slot(b) + size_t(row) * head_row_bytes;
              float acc[4] = {0.f, 0.f, 0.f, 0.f};
              auto acc8 = [&](const float (&f)[8], const float* x) {
                acc[0] = fmaf(f[0], x[0], acc[0]); acc[1] = fmaf(f[1], x[1], acc[1]);
                acc[2] = fmaf(f[2], x[2], acc[2]); acc[3] = fmaf(f[3], x[3], acc[3]);
                acc[0] = fmaf(f[4], x[4], acc[0]); acc[1] = fmaf(f[5], x[5], acc[1]);
                acc[2] = fmaf(f[6], x[6], acc[2]); acc[3] = fmaf(f[7], x[7], acc[3]);
              };
#pragma unroll
              for (int m = 0; m < kHV; ++m) {
                if (lane + 32 * m < hn) {
                  float f[8];
                  if (q8) i8x8_to_float(reinterpret_cast<const uint2*>(wrow)[lane + 32 * m], f);
                  else f16x8(reinterpret_cast<const uint4*>(wrow)[lane + 32 * m], f);
                  acc8(f, xr[m]);
                }
              }
              for (int c = lane + 32 * kHV; c < hn; c += 32) {   // rows wider than kHV groups per lane
                float f[8];
                if (q8) i8x8_to_float(reinterpret_cast<const uint2*>(wrow)[c], f);
                else f16x8(reinterpret_cast<const uint4*>(wrow)[c], f);
                acc8(f, xn + c * 8);
              }
              float lg = warp_sum((acc[0] + acc[1]) + (acc[2] + acc[3]));
              if (lane == 0) {
                if (q8) lg *= sc[rsub];
                if (a.logits) a.logits[r0 + row] = lg;
                if (lg > best || (lg == best && r0 + row < besti)) {
                  best = lg;
                  besti = r0 + row;
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(empty_h + b);      // this warp is done with the slot
        }
        PT(PH_HEAD_STREAM);
        // best of each warp, then of the CTA
        if (lane == 0) {
          scratch32[2 * warp] = __float_as_uint(best);
          scratch32[2 * warp + 1] = uint32_t(besti);
        }
        alive = csync_and(hok) && alive;
        if (tid == 0) {
          float bv = -INFINITY;
          int bi = 0x7fffffff;
          for (int i = 0; i < kPWarps; ++i) {
            const float v = __uint_as_float(scratch32[2 * i]);
            const int id = int(scratch32[2 * i + 1]);
            if (v > bv || (v == bv && id < bi)) { bv = v; bi = id; }
          }
          tw_put(a.x_head + 2 * w.c, __float_as_uint(bv), tag(L, XHEAD));
          tw_put(a.x_head + 2 * w.c + 1, uint32_t(bi), tag(L, XHEAD));
        }
        csync();
        if (w.c == 0 && alive) {
          if (tw_gather<1>(status, ctl, a.x_head, 2 * G, scratch32, a.x_head, 0, scratch32, tag(L, XHEAD), 2048u) &&
              tid == 0) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
            for (int c = 0; c < G; ++c) {
              const float v = __uint_as_float(scratch32[2 * c]);
              const int id = int(scratch32[2 * c + 1]);
              if (v > bv || (v == bv && id < bi)) { bv = v; bi = id; }
            }
            a.tok_out[0] = bi == 0x7fffffff ? 0 : bi;
          }
        }
      }
      PT(PH_HEAD_ARG);
    }
#ifdef DFSSM_PHASE_TIMERS
    if (tid == 0 && a.phase) {
      for (int i = 0; i < PH_N; ++i) a.phase[size_t(w.c) * kPhaseSlots + i] += ptime[i];
      a.phase[size_t(w.c) * kPhaseSlots + kPhaseSlots - 1] += 1;   // calls
    }
#endif
#undef PT
    // ---- end of token: CTA 0 advances the launch epoch once every CTA has
    // published into the last exchange (so all have read the epoch)
    if (w.c == 0 && tid == 0 && !aborted(ctl)) ctl[0] = ctl[0] + 1;
    // after an abort, give copies that other CTAs may still have in flight towards
    // this CTA time to land before the cluster lets it exit
    if (aborted(ctl)) {
      const long long t0 = clock64();
      while (clock64() - t0 < 200000) __nanosleep(1000);
    }
  }
  __syncwarp();
  // no CTA leaves while another CTA of its cluster may still write into it
  cluster_sync_all();
}
#undef PSM

// ------------------------------------------------------------------ host side

inline size_t persistent_exchange_words(int D, int E, int grid) { return size_t(D) + E + 6 * size_t(grid); }

inline size_t persistent_scratch_bytes(int batch, int d_model, int d_inner, int in_rows, int head_blocks) {
  (void)in_rows;
  // multi-launch LM-head partials + persistent control words + exchange words (upper bounds)
  const size_t head = size_t(8) * (batch > 0 ? batch : 1) * (head_blocks > 0 ? head_blocks : 1);
  const size_t words = persistent_exchange_words(d_model, d_inner, 1024);
  return head + 256 + 8 * words + 256;
}

}  // namespace dfssm
