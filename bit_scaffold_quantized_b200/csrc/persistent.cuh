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
// The layer is instruction-bound, so no CTA repeats work that its cluster can
// split: every activation vector is prepared in Q slices (CTA of rank r owns
// columns [r S, (r+1) S)), and the cluster all-gathers the slices' scaffold digit
// planes, their integer sums and their max |x| with bulk copies from shared memory
// into the other CTAs' shared memory (completion counted in bytes on the
// receiver's mbarrier).  LoRA stage 1 is split the same way (each CTA multiplies
// its slice of the int8 codes with its slice of every A row; the int32 partials
// are all-gathered and summed in a fixed order, so the result is exact).
//
// Grid-wide exchanges (two per layer) go through "tagged words" in global memory:
// 64-bit words holding 32 data bits and a 32-bit tag (launch epoch, layer,
// exchange kind), stored and polled without fences; a word is valid exactly when
// its tag matches.  Besides the values, each producer publishes the fp64 sum of
// squares of its values, so a consumer of a slice still gets the full RMSNorm.
//
// Per layer (B = 1), CTA c of cluster k, rank r:
//   R    gather slice r of the residual and the sum-of-squares partials
//   A    x = fp16(rmsnorm(res) w) on the slice: digit planes, sum, max -> cluster
//   B    int8 codes of the slice, LoRA partials of all rows -> cluster
//   -    exact int8 scaffold MMA on its in_proj tiles: the z and x rows of its own
//        SSM channels plus its share of the cluster's "shared" tiles (all B/C rows
//        and the dt rows of the cluster's heads; every cluster computes them)
//   C    LoRA stage 2, conv step of its x channels; shared rows (B/C after conv +
//        SiLU, raw dt) -> cluster
//   G    SSM update of its own state rows, g = y silu(z) and its sum of squares
//        published as fp32 / fp64 tagged words
//   A'B' the gated RMSNorm, codes and LoRA stage 1 of the out_proj on slice r of g
//   R'   out_proj rows of its tiles added to the residual and published
// Final: gather the residual, final RMSNorm, stream this CTA's LM-head rows,
// publish (best logit, id); CTA 0 reduces to the greedy token.
//
// Every spin is bounded: a wait that gives up sets a status bit and an abort flag
// that makes every CTA leave the token early; all CTAs of a cluster meet at a
// final cluster barrier (after an abort, only once in-flight copies have had time
// to land), so none exits while another may still write into it.
#pragma once

#include "common.cuh"

namespace dfssm {

constexpr int kMaxLayers = 64;
constexpr int kPWarps = 15;                       // compute warps
constexpr int kPThreads = 32 * kPWarps;           // compute threads
constexpr int kPBlock = kPThreads + 32;           // + the copy warp: 16 warps, 128 registers each
constexpr int kPMaxUnits = 3;                     // SSM row units (16 channels) per CTA
constexpr int kPMaxShared = 4;                    // shared (B/C, dt) tiles per CTA
constexpr int kPMaxInTiles = 8;                   // z, x and shared tiles per CTA
constexpr int kPMaxSharedTiles = 20;              // shared tiles of one cluster
constexpr int kPMaxSharedRows = 16 * kPMaxSharedTiles;
constexpr int kPMaxOutTiles = 2;                  // out_proj tiles per CTA
constexpr int kPMaxCluster = 8;
constexpr int kPMaxHeads = 4;                     // heads touched by one CTA's SSM rows
constexpr int kPSsmRows = (kPMaxUnits * 16 + kPWarps - 1) / kPWarps;   // SSM rows per compute warp
constexpr long long kSpinLimit = 1LL << 22;       // polls before a wait gives up (seconds)
constexpr int kHeadChunkRows = 7;                  // LM-head rows per chunk: 14 warps = 7 rows x 2 halves
constexpr int kHeadRingMax = 8;                   // LM-head chunk slots (all buffers free after the last layer)

// tagged-word exchange kinds
enum { XR = 0, XG = 1, XHEAD = 2 };
// cluster exchanges (one mbarrier each, one phase per layer)
enum { EX_A_IN = 0, EX_B_IN = 1, EX_C = 2, EX_A_OUT = 3, EX_B_OUT = 4, EX_N = 5 };

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
  int vs, xs, xqs, stg_a, asm_a, stg_b, rcv_b, yin, shr, stg_c, shst, u, resown;
  int ring_end, head_slots;       // LM-head chunk slots [0, head_slots) tile [0, ring_end)
  int part, full, misc;
  int total;
};

struct __align__(16) PParams {
  // shape
  int n_layer, D, E, H, P, N, R, in_rows, C, vocab;
  int kg_in, kg_out;             // 256-column groups of the in/out projections
  int units, grid, Q;            // SSM row units (E/16), CTAs, CTAs per cluster
  int n_bc_tiles, dt_tile0;      // 2N/16 and first dt tile index
  int out_tiles;                 // D/16
  int SD, SE, lgSD, lgSE;        // slice widths (D/Q, E/Q, powers of two) and their log2
  int BSD, BSE;                  // bytes of one slice block: 6 digit planes (+16 pad each) + sum + max
  int layer_mode;                // 1: residual in/out from `residual`, no embedding / head
  PSmem sm;
  // io
  const uint16_t* embed; const uint16_t* normf_w; const int32_t* tok_in; int32_t* tok_out; float* logits;
  const int8_t* embed_q;         // int8 per-row embedding (replaces embed when not null)
  const float* embed_s;          // its fp32 row scales
  float* residual;               // layer mode: [D] in/out
  // workspace
  unsigned* status;              // status word
  unsigned* ctl;                 // [0] launch epoch, [1] abort flag
  unsigned long long* x_r;       // D residual words
  unsigned long long* x_rs;      // 2 grid words: fp64 sum of squares of each CTA's residual rows
  unsigned long long* x_g;       // E gated-value words
  unsigned long long* x_gs;      // 2 grid words: fp64 sum of squares of each CTA's gated values
  unsigned long long* x_head;    // 2 grid words
  // diagnostics of the last layer (workspace regions of dfssm_ws_layout)
  uint16_t* d_x_in; int8_t* d_xq_in; float* d_sx_in; int* d_acc_in; double* d_u_in; int8_t* d_xd_in;
  int* d_xdsum_in; double* d_zx; double* d_xc; float* d_g; uint16_t* d_x_out; int8_t* d_xq_out;
  float* d_sx_out; int* d_acc_out; double* d_u_out; int8_t* d_xd_out; int* d_xdsum_out; float* d_res;
  PLayer L[kMaxLayers];
};


// Shared-memory plan of one shape (byte offsets); the host plans launches with the
// same function, and the compile-time shape below bakes its result into the code.
constexpr int kPlanSMs = 256;   // upper bound on CTAs of one launch (sizes the exchange scratch)

__host__ __device__ constexpr int ptake(int& off, int bytes) {
  const int at = off;
  off = (off + (bytes > 16 ? bytes : 16) + 15) & ~15;
  return at;
}

__host__ __device__ constexpr PSmem plan_smem(int D, int E, int H, int N, int R, int Q) {
  PSmem m{};
  const int kg_in = D / kTileCols, kg_out = E / kTileCols;
  const int SD = D / Q, SE = E / Q;
  const int BSD = kDigits * (SD + 16) + 16, BSE = kDigits * (SE + 16) + 16;
  const int Smax = SD > SE ? SD : SE, BSmax = BSD > BSE ? BSD : BSE, R4 = R > 4 ? R : 4, R1 = R > 1 ? R : 1;
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
  m.prenorm = ptake(off, 2 * SD);
  m.sa_in = ptake(off, 2 * R);
  m.hd_dtb = ptake(off, 4 * H);
  m.hd_alog = ptake(off, 4 * H);
  m.hd_d = ptake(off, 4 * H);
  m.state = ptake(off, kPMaxUnits * 16 * N * 4);
  m.ab_end = off;
  m.out_tiles = ptake(off, kPMaxOutTiles * kg_out * 512);
  m.out_bq = ptake(off, kPMaxOutTiles * 16 * R);
  m.out_alpha = ptake(off, kPMaxOutTiles * 32);
  m.out_sb = ptake(off, kPMaxOutTiles * 32);
  m.a_out = ptake(off, R * SE);
  m.gnorm = ptake(off, 2 * SE);
  m.sa_out = ptake(off, 2 * R);
  m.cd_end = off;
  m.vs = ptake(off, 4 * Smax);
  m.xs = ptake(off, 2 * Smax);
  m.xqs = ptake(off, Smax);
  m.stg_a = ptake(off, BSmax);
  m.asm_a = ptake(off, Q * BSmax);
  m.stg_b = ptake(off, 4 * R4);
  m.rcv_b = ptake(off, Q * 4 * R4);
  m.yin = ptake(off, kPMaxInTiles * 16 * 8);
  m.shr = ptake(off, 2 * kPMaxSharedRows * 8);
  m.stg_c = ptake(off, 2 * kPMaxShared * 16 * 8);
  m.shst = ptake(off, 3 * kPMaxShared * 16 * 4);
  m.u = ptake(off, 8 * R1);
  m.resown = ptake(off, kPMaxOutTiles * 16 * 4);
  // everything above is free once the last layer is done: the LM-head chunk ring
  // (grown to five chunks when that still leaves room for the rest)
  const int chunk = kHeadChunkRows * 2 * D;
  if (off < 5 * chunk && 5 * chunk + 4 * (2 * kPlanSMs + 2 * D) + 8 * 1024 <= 200 * 1024) off = 5 * chunk;
  m.ring_end = off;
  m.head_slots = off / chunk;
  if (m.head_slots > kHeadRingMax) m.head_slots = kHeadRingMax;
  m.part = ptake(off, 16 * 16 * kDigits * 4);
  m.full = ptake(off, 4 * (2 * kPlanSMs + 2 * D));
  m.misc = ptake(off, kPMaxInTiles * 16 * 8);
  m.total = off;
  return m;
}

// Shapes: the kernel reads every size and shared-memory offset either from its
// parameters (any eligible shape) or from compile-time constants (the shape of the
// 48-layer, d_model 2048 model; address arithmetic then folds into immediates).
struct ShapeAny {
  static constexpr bool kConst = false;
  static constexpr int D = 0, E = 0, H = 0, P = 0, N = 0, R = 0, Q = 0, C = 0, kg_in = 0, kg_out = 0;
  static constexpr int SD = 0, SE = 0, lgSD = 0, lgSE = 0, BSD = 0, BSE = 0;
  static constexpr int units = 0, n_bc_tiles = 0, dt_tile0 = 0, out_tiles = 0;
  static constexpr PSmem kPlan{};
};
struct Shape2048 {
  static constexpr bool kConst = true;
  static constexpr int D = 2048, E = 4096, H = 64, P = 64, N = 128, R = 32, Q = 8, C = E + 2 * N;
  static constexpr int kg_in = D / kTileCols, kg_out = E / kTileCols;
  static constexpr int SD = D / Q, SE = E / Q, lgSD = 8, lgSE = 9;
  static constexpr int BSD = kDigits * (SD + 16) + 16, BSE = kDigits * (SE + 16) + 16;
  static constexpr int units = E / 16, n_bc_tiles = 2 * N / 16, dt_tile0 = (2 * E + 2 * N) / 16, out_tiles = D / 16;
  static constexpr PSmem kPlan = plan_smem(D, E, H, N, R, Q);
};
static_assert((1 << Shape2048::lgSD) == Shape2048::SD && (1 << Shape2048::lgSE) == Shape2048::SE, "slice widths");

// ------------------------------------------------------------------ primitives

DFSSM_DEV bool mbar_try_wait_cluster(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Shared memory of this CTA -> shared memory of a CTA of the cluster (addresses
// from cluster_map), completion counted on that CTA's mbarrier.
DFSSM_DEV void bulk_s2c(uint32_t dst, const void* src, unsigned bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :: "r"(dst), "r"(smem_u32(src)), "r"(bytes), "r"(bar) : "memory");
}
// Named barrier 1 over the CTA's 16 warps.
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

DFSSM_DEV void give_up(unsigned* status, unsigned* ctl, unsigned bit) {
  atomicOr(status, bit);
  atomicExch(ctl + 1, 1u);
}

// Compute warps: gather n1 tagged words from src1 into dst1 and n2 from src2 into
// dst2 (32-bit payloads).  Returns false (after flagging) if a word did not arrive
// within the spin limit.
DFSSM_DEV bool tw_gather2(unsigned* status, unsigned* ctl, const unsigned long long* src1, int n1, uint32_t* dst1,
                          const unsigned long long* src2, int n2, uint32_t* dst2, uint32_t tag, unsigned bit) {
  bool ok = true;
  const int n = n1 + n2;
  for (int base = 0; base < n && ok; base += 4 * kPThreads) {
    unsigned long long w[4];
    int idx[4];
    unsigned pending = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      idx[i] = base + i * kPThreads + int(threadIdx.x);
      if (idx[i] < n) pending |= 1u << i;
    }
    long long spins = 0;
    while (pending) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (pending & (1u << i)) w[i] = tw_load(idx[i] < n1 ? src1 + idx[i] : src2 + (idx[i] - n1));
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if ((pending & (1u << i)) && uint32_t(w[i] >> 32) == tag) {
          *(idx[i] < n1 ? dst1 + idx[i] : dst2 + (idx[i] - n1)) = uint32_t(w[i]);
          pending &= ~(1u << i);
        }
      if (pending && ((++spins & 255) == 0) && (spins > kSpinLimit || aborted(ctl))) {
        give_up(status, ctl, bit);
        ok = false;
        break;
      }
    }
  }
  return csync_and(ok);
}

// Bounded wait by one thread.
DFSSM_DEV bool mbar_wait(unsigned* status, unsigned* ctl, uint64_t* bar, unsigned parity, unsigned bit) {
  long long spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if (((++spins & 255) == 0) && (spins > kSpinLimit || aborted(ctl))) {
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
// this CTA and waits (bounded) for the phase, the compute warps agree, then every
// thread takes the phase once more to acquire the cluster's writes for itself.
DFSSM_DEV bool xwait(unsigned* status, unsigned* ctl, uint64_t* bar, unsigned bytes, unsigned parity, unsigned bit) {
  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_expect_tx(bar, bytes);
    long long spins = 0;
    while (!mbar_try_wait_cluster(bar, parity)) {
      if (((++spins & 255) == 0) && (spins > kSpinLimit || aborted(ctl))) {
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
// Send `bytes` of this CTA's staging buffer to offset `dst` (same layout in every
// CTA) of every CTA of the cluster.  The writing threads have already fenced their
// stores for the async proxy; the compute warps meet once so the copies see them.
DFSSM_DEV void xsend(const void* stage, void* dst, unsigned bytes, uint64_t* bar, int Q) {
  csync();
  if (int(threadIdx.x) < Q && bytes > 0)
    bulk_s2c(cluster_map(smem_u32(dst), threadIdx.x), stage, bytes, cluster_map(smem_u32(bar), threadIdx.x));
}

// Compute-warp reductions (fixed order, identical in every CTA).
DFSSM_DEV double csum_d(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_d(v);
  if (lane == 0) red[warp] = v;
  csync();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kPWarps; ++w) t += red[w];
  csync();
  return t;
}
// Sum of the fp64 partials published by the grid's CTAs (word pairs), in CTA order,
// by warp 0; every compute thread gets the result.
DFSSM_DEV double sum_partials(const uint32_t* words, int G, double* red) {
  const int lane = threadIdx.x & 31;
  if ((threadIdx.x >> 5) == 0) {
    double t = 0.0;
    for (int c = lane; c < G; c += 32) t += f64_of(words + 2 * c);
    t = warp_sum_d(t);
    if (lane == 0) red[0] = t;
  }
  csync();
  const double v = red[0];
  csync();
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
// its slice of every LoRA A row and of the pre-norm weight, its SSM state rows and
// the conv weights and state of its x channels and B/C rows.
DFSSM_DEV void produce_ab(const PParams& a, const PWork& w, const PLayer& L, unsigned char* sm, uint64_t* full) {
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
    c.put(s.prenorm, L.prenorm_w + size_t(w.r) * a.SD, 2 * a.SD);
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
// scales, its slice of every LoRA A row and of the gated-norm weight.
DFSSM_DEV void produce_cd(const PParams& a, const PWork& w, const PLayer& L, unsigned char* sm, uint64_t* full) {
  const PSmem& s = a.sm;
  issue_group(sm, full, [&](CopyList& c) {
    const int tile_bytes = a.kg_out * 512;
    c.put(s.gnorm, L.gnorm_w + size_t(w.r) * a.SE, 2 * a.SE);
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

// Slice preparation (elements tid, tid + kPThreads, ...): x = fp16((v rs) w) into
// xs, its six digit planes into the staging block (plane stride S + 16), and the
// block tail: the exact sum of the slice's X = x 2^24 (int64) and max |x| (fp16 bits).
DFSSM_DEV void prep_slice(const float* v, const uint16_t* w, int S, double rs, unsigned char* stage, int* red,
                          uint16_t* xs, uint16_t* x_diag, int8_t* xd_diag, int K_diag) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int PS = S + 16;
  const float rs32 = float(rs);
  int xh = 0, xl = 0;
  unsigned am = 0;
  for (int i = tid; i < S; i += kPThreads) {
    const uint32_t h = norm_fp16(v[i], rs, rs32, half_to_float_bits(w[i]));
    uint32_t lo, hi;
    digits_of(h, &lo, &hi);
    xs[i] = uint16_t(h);
    stage[i] = uint8_t(lo);
    stage[PS + i] = uint8_t(lo >> 8);
    stage[2 * PS + i] = uint8_t(lo >> 16);
    stage[3 * PS + i] = uint8_t(lo >> 24);
    stage[4 * PS + i] = uint8_t(hi);
    stage[5 * PS + i] = uint8_t(hi >> 8);
    const long long X = half_times_2p24_64(h);
    xh += int(X >> 20);                      // X = xh 2^20 + xl, 0 <= xl < 2^20
    xl += int(X & 0xfffff);
    am = max(am, h & 0x7fffu);
    if (x_diag) {
      x_diag[i] = uint16_t(h);
      xd_diag[i] = int8_t(lo);
      xd_diag[K_diag + i] = int8_t(lo >> 8);
      xd_diag[2 * K_diag + i] = int8_t(lo >> 16);
      xd_diag[3 * K_diag + i] = int8_t(lo >> 24);
      xd_diag[4 * K_diag + i] = int8_t(hi);
      xd_diag[5 * K_diag + i] = int8_t(hi >> 8);
    }
  }
  // per thread |xh|, xl < 2^21: 32-lane sums fit int32; the warps' sums are combined in int64
  const int sh = __reduce_add_sync(0xffffffffu, xh);
  const int sl = __reduce_add_sync(0xffffffffu, xl);
  const unsigned amw = __reduce_max_sync(0xffffffffu, am);
  if (lane == 0) {
    red[3 * warp] = sh;
    red[3 * warp + 1] = sl;
    red[3 * warp + 2] = int(amw);
  }
  csync();
  if (tid == 0) {
    long long sum = 0;
    unsigned mx = 0;
    for (int i = 0; i < kPWarps; ++i) {
      sum += (static_cast<long long>(red[3 * i]) << 20) + red[3 * i + 1];
      mx = max(mx, unsigned(red[3 * i + 2]));
    }
    *reinterpret_cast<long long*>(stage + kDigits * PS) = sum;
    *reinterpret_cast<unsigned*>(stage + kDigits * PS + 8) = mx;
  }
  fence_async_smem();
}

// After the cluster's slice blocks arrived: exact sum of X over the whole vector
// and its max |x| (fp16 bits), in a fixed order.
DFSSM_DEV void slice_totals(const unsigned char* asmb, int Q, int S, int BS, long long* xsum, unsigned* amax) {
  long long s = 0;
  unsigned m = 0;
  for (int q = 0; q < Q; ++q) {
    const unsigned char* t = asmb + q * BS + kDigits * (S + 16);
    s += *reinterpret_cast<const long long*>(t);
    m = max(m, *reinterpret_cast<const unsigned*>(t + 8));
  }
  *xsum = s;
  *amax = m;
}

// Digit-plane sums of the whole vector from the cluster's blocks (diagnostics only),
// by all compute threads.
DFSSM_DEV void plane_sums(const unsigned char* asmb, int Q, int S, int BS, int* red, int* out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int d = 0; d < kDigits; ++d) {
    int t = 0;
    for (int i = tid; i < Q * S; i += kPThreads) t += int(int8_t(asmb[(i / S) * BS + d * (S + 16) + i % S]));
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

// int8 codes of the slice (from its fp16 bits), then LoRA stage-1 partials of the
// slice for all R rows: stage[j] = sum_k A[j][k] q[k] over the slice, fenced for the
// async proxy.
DFSSM_DEV void codes_and_lora_partials(const uint16_t* xs, int S, float sx, float rcp, bool nonzero, int8_t* xqs,
                                       const int8_t* Aslice, int R, int* stage, int8_t* xq_diag) {
  const int tid = threadIdx.x;
  for (int i = tid; i < S; i += kPThreads) {
    const int q = nonzero ? quant_code_bits(half_to_float_bits(xs[i]), sx, rcp) : 0;
    xqs[i] = int8_t(q);
    if (xq_diag) xq_diag[i] = int8_t(q);
  }
  csync();
  if (R > 0) {
    // 16 lanes per row, two rows per warp; rows beyond the first pass of the warps
    // come round again
    const int half = (tid & 31) >> 4, sub = tid & 15;
    for (int j = 2 * (tid >> 5) + half; j < R; j += 2 * kPWarps) {
      const int* A4 = reinterpret_cast<const int*>(Aslice + j * S);
      const int* q4 = reinterpret_cast<const int*>(xqs);
      int acc = 0;
      for (int i = sub; i < S / 4; i += 16) acc = __dp4a(A4[i], q4[i], acc);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (sub == 0) {
        stage[j] = acc;
        fence_async_smem();
      }
    }
  }
}

// Sum of the cluster's LoRA partials (fixed order) -> u[j] = acc sA[j] sx in fp64.
DFSSM_DEV void lora_finish(const int* rcv, int Q, int R, const uint16_t* sA, float sx, double* u, int* acc_diag,
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

// LoRA stage 2 for `nrows` rows: out[r] = sum_j B[r][j] u[j] in fp64, one thread
// per row with four interleaved partial sums (R is a multiple of 8).
DFSSM_DEV void lora2_rows(const int8_t* Bq, int nrows, const double* u, int R, double* out) {
  for (int r = threadIdx.x; r < nrows; r += kPThreads) {
    const int* b4 = reinterpret_cast<const int*>(Bq + r * R);
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int j4 = 0; j4 < R / 4; ++j4) {
      const int v = b4[j4];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = fma(double(int8_t(v >> (8 * e))), u[4 * j4 + e], acc[e]);
    }
    out[r] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  }
}

// Exact scaffold MMA over `ntile` tiles (smem, kg groups each), split into units
// (tile, kgroup chunk); int32 partials to part[unit][16][kDigits].  The activation
// digit planes come from the cluster's slice blocks: column k lies in block
// k >> lgS at offset k & (S - 1) of each plane (stride S + 16).  Register q of the
// A fragment of product s is word q of the lane's sign vector masked to bits
// s, s + 8, s + 16, s + 24: unsigned bytes 0 or 2^s, one instruction per register.
// Product s accumulates into its own set, 2^s times its 0/1 sums (|sum| < 2^27),
// and the sets are recombined exactly with right shifts.  One 16-byte load per
// plane row gives the B fragments of products 2m and 2m + 1.  Returns the chunks
// per tile.
DFSSM_DEV int scaffold_mma(const unsigned char* tiles, int ntile, int kg, const unsigned char* asmb, int lgS, int BS,
                           int* part) {
  constexpr int nw = kPWarps;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  int nchunk = nw / ntile;
  if (nchunk < 1) nchunk = 1;
  if (nchunk > kg) nchunk = kg;
  const int S = 1 << lgS;
  const int nunits = ntile * nchunk;
  const unsigned char* dbase = asmb + (g < kDigits ? g : 0) * (S + 16);
  for (int unit = warp; unit < nunits; unit += nw) {
    const int ti = unit / nchunk, ci = unit % nchunk;
    const int kg_lo = ci * kg / nchunk, kg_hi = (ci + 1) * kg / nchunk;
    int acc[8][4];
#pragma unroll
    for (int s = 0; s < 8; ++s) acc[s][0] = acc[s][1] = acc[s][2] = acc[s][3] = 0;
    const uint4* tw = reinterpret_cast<const uint4*>(tiles + size_t(ti) * kg * 512);
    for (int kgi = kg_lo; kgi < kg_hi; ++kgi) {
      const uint4 wv = tw[kgi * 32 + lane];
      const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        // 16 aligned columns never straddle a slice block (S >= 16)
        const int k0 = kgi * kTileCols + 64 * m + 16 * t;
        uint4 bq = make_uint4(0, 0, 0, 0);
        if (g < kDigits) bq = *reinterpret_cast<const uint4*>(dbase + (k0 >> lgS) * BS + (k0 & (S - 1)));
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t mask = 0x01010101u << (2 * m + e);
          const uint32_t af[4] = {words[0] & mask, words[1] & mask, words[2] & mask, words[3] & mask};
          mma_u8s8_16832(acc[2 * m + e], af, e ? bq.z : bq.x, e ? bq.w : bq.y);
        }
      }
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

// Scaffold value (without alpha) of row r of tile ti from the unit partials:
// sum_k s_k x_k = 2^-24 (2 sum_d 256^d Q_d - sum_k X_k), exact in int64.
DFSSM_DEV double tile_row_value(const int* part, int ti, int nchunk, int r, long long xsum) {
  long long S = 0;
#pragma unroll
  for (int d = kDigits - 1; d >= 0; --d) {
    int s = 0;
    for (int c = 0; c < nchunk; ++c) s += part[((ti * nchunk + c) * 16 + r) * kDigits + d];
    S = S * 256 + s;
  }
  return double(2 * S - xsum) * (1.0 / 16777216.0);
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
  __shared__ double ssw[kPWarps * kPSsmRows];
  for (int i = threadIdx.x; i < int(sizeof(PParams) / 16); i += blockDim.x)
    reinterpret_cast<uint4*>(pbuf)[i] = reinterpret_cast<const uint4*>(&pa)[i];
  const PParams& a = *reinterpret_cast<const PParams*>(pbuf);
  const PWork w = assign(pa);
  // sizes: compile-time for a fixed shape, else from the parameters
  constexpr bool kC = SH::kConst;
  const int D = kC ? SH::D : pa.D, E = kC ? SH::E : pa.E, P = kC ? SH::P : pa.P, N = kC ? SH::N : pa.N;
  const int R = kC ? SH::R : pa.R, C = kC ? SH::C : pa.C, Q = kC ? SH::Q : pa.Q;
  const int kg_in = kC ? SH::kg_in : pa.kg_in, kg_out = kC ? SH::kg_out : pa.kg_out;
  const int SD = kC ? SH::SD : pa.SD, SE = kC ? SH::SE : pa.SE, lgSD = kC ? SH::lgSD : pa.lgSD;
  const int lgSE = kC ? SH::lgSE : pa.lgSE, BSD = kC ? SH::BSD : pa.BSD, BSE = kC ? SH::BSE : pa.BSE;
#define PSM(f) (kC ? SH::kPlan.f : pa.sm.f)
  uint64_t* full_ab = &bars[0];
  uint64_t* empty_ab = &bars[1];
  uint64_t* full_cd = &bars[2];
  uint64_t* empty_cd = &bars[3];
  uint64_t* full_h = &bars[4];
  uint64_t* empty_h = &bars[4 + kHeadRingMax];
  __shared__ int s_stale;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4 + 2 * kHeadRingMax; ++i) mbar_init(&bars[i], 1);
    for (int i = 0; i < EX_N; ++i) mbar_init(&xbars[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // An abort flag left by an earlier call means its exchange words may still carry
    // this launch's epoch: do nothing and say so (the caller zero-fills the workspace).
    s_stale = aborted(pa.ctl) ? 1 : 0;
    if (s_stale) atomicOr(pa.status, 1u);
  }
  // every CTA's barriers exist before any CTA of the cluster copies into it
  cluster_sync_all();
  const bool stale = s_stale != 0;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.grid;
  const int v0 = int((long long)w.c * a.vocab / G), v1 = int((long long)(w.c + 1) * a.vocab / G);
  // LM-head rows: fp16, or (Q8) int8 codes with a per-row scale.  Slots are spaced for
  // 7 fp16 rows, which is 14 int8 rows: an int8 chunk is 14 rows (half the chunks).
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

    float* vs = sp<float>(sm, PSM(vs));                 // this CTA's slice of the residual / gated value
    uint16_t* xs = sp<uint16_t>(sm, PSM(xs));          // fp16 bits of this CTA's slice
    int8_t* xqs = sp<int8_t>(sm, PSM(xqs));
    unsigned char* stg_a = sm + PSM(stg_a);            // own slice block
    unsigned char* asm_a = sm + PSM(asm_a);            // the cluster's slice blocks
    int* stg_b = sp<int>(sm, PSM(stg_b));              // own LoRA partials
    int* rcv_b = sp<int>(sm, PSM(rcv_b));              // the cluster's LoRA partials
    int* part = sp<int>(sm, PSM(part));
    double* yin = sp<double>(sm, PSM(yin));            // [kPMaxInTiles * 16] in_proj outputs of own tiles (slot order)
    double* shr = sp<double>(sm, PSM(shr));            // [kPMaxSharedRows] the cluster's shared rows
    double* stg_c = sp<double>(sm, PSM(stg_c));        // own shared rows
    float* shst = sp<float>(sm, PSM(shst));            // [3][kPMaxShared * 16] new conv state of own B/C rows
    double* u = sp<double>(sm, PSM(u));                // [R] LoRA stage-1 outputs
    float* resown = sp<float>(sm, PSM(resown));        // residual of own out_proj rows
    double* lo = sp<double>(sm, PSM(misc));            // LoRA stage-2 sums of own rows
    uint32_t* scratch32 = sp<uint32_t>(sm, PSM(full));
    const int zslot = 0, xslot = w.nu, shslot = 2 * w.nu;
    const int SHR = kPMaxShared * 16;
    const int r0D = w.r * SD, r0E = w.r * SE;   // this CTA's slices

    // ---- layer-0 residual: own slice, own out rows, sum of squares (every CTA)
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
      auto res0 = [&](int k) {
        return a.layer_mode ? a.residual[k] : q8 ? es * float(eqrow[k]) : h2f(erow[k]);
      };
      double acc = 0.0;
      for (int k = tid; k < D; k += kPThreads) {
        const double v = double(res0(k));
        acc = fma(v, v, acc);
      }
      for (int k = tid; k < SD; k += kPThreads) vs[k] = res0(r0D + k);
      if (tid < w.no * 16) resown[tid] = res0(w.o0 * 16 + tid);
      ss = csum_d(acc, redd);
    }

    bool alive = true;
    for (int l = 0; l < a.n_layer && alive; ++l) {
      const PLayer& L = a.L[l];
      const bool diag = (l == a.n_layer - 1);
      const bool cdiag = diag && w.k == 0;      // cluster 0 writes the slice diagnostics
      const bool wdiag = diag && w.c == 0;
      const unsigned par = unsigned(l) & 1u;

      // ---- R: own slice of the residual and the sums of squares
      if (l > 0) {
        if (!tw_gather2(status, ctl, a.x_r + r0D, SD, reinterpret_cast<uint32_t*>(vs), a.x_rs, 2 * G, scratch32,
                        tag(l, XR), 4u)) {
          alive = false;
          break;
        }
        ss = sum_partials(scratch32, G, redd);
      }
      if (!mbar_wait_compute(status, ctl, full_ab, par, 8u)) { alive = false; break; }

      // ---- A: pre-norm on the slice -> the cluster
      const double rs_in = 1.0 / sqrt(ss / double(D) + kEpsD);
      prep_slice(vs, sp<uint16_t>(sm, PSM(prenorm)), SD, rs_in, stg_a, redi, xs, cdiag ? a.d_x_in + r0D : nullptr,
                 cdiag ? a.d_xd_in + r0D : nullptr, D);
      xsend(stg_a, asm_a + w.r * BSD, unsigned(BSD), &xbars[EX_A_IN], Q);
      if (!xwait(status, ctl, &xbars[EX_A_IN], unsigned(Q * BSD), par, 16u)) { alive = false; break; }
      long long xsum_in;
      unsigned amax_in;
      slice_totals(asm_a, Q, SD, BSD, &xsum_in, &amax_in);
      const float am_in = half_to_float_bits(amax_in);
      const float sx_in = am_in > 0.f ? __fdiv_rn(am_in, 127.f) : 1.f;
      if (wdiag) {
        if (tid == 0) *a.d_sx_in = sx_in;
        plane_sums(asm_a, Q, SD, BSD, redi, a.d_xdsum_in);
      }
      // ---- B: codes and LoRA partials of the slice -> the cluster
      codes_and_lora_partials(xs, SD, sx_in, __frcp_rn(sx_in), am_in > 0.f, xqs, sp<int8_t>(sm, PSM(a_in)), R,
                              stg_b, cdiag ? a.d_xq_in + r0D : nullptr);
      if (R) xsend(stg_b, rcv_b + w.r * R, unsigned(4 * R), &xbars[EX_B_IN], Q);
      // ---- in_proj scaffold on own tiles
      const int nch_in = scaffold_mma(sm + PSM(in_tiles), w.ntile, kg_in, asm_a, lgSD, BSD, part);
      if (tid < w.ntile * 16)
        yin[tid] = h2d(sp<uint16_t>(sm, PSM(in_alpha))[tid]) * tile_row_value(part, tid / 16, nch_in, tid % 16, xsum_in);
      // ---- u_in, LoRA stage 2 of own rows
      if (R) {
        if (!xwait(status, ctl, &xbars[EX_B_IN], unsigned(Q * 4 * R), par, 32u)) { alive = false; break; }
        lora_finish(rcv_b, Q, R, sp<uint16_t>(sm, PSM(sa_in)), sx_in, u, wdiag ? a.d_acc_in : nullptr, a.d_u_in);
        lora2_rows(sp<int8_t>(sm, PSM(in_bq)), w.ntile * 16, u, R, lo);
      }
      csync();
      if (tid < w.ntile * 16) {
        double y = yin[tid];
        if (R) y = fma(h2d(sp<uint16_t>(sm, PSM(in_sb))[tid]), lo[tid], y);
        yin[tid] = y;
        if (diag) a.d_zx[slot_tile(a, w, tid / 16) * 16 + tid % 16] = y;
      }
      csync();
      // ---- C: conv step of own x channels, gate, shared rows -> the cluster
      if (tid < w.nu * 16) {
        const int uu = tid / 16, r = tid % 16;
        const double xv = yin[(xslot + uu) * 16 + r];
        const uint16_t* cw = sp<uint16_t>(sm, PSM(convw_x)) + (uu * 16 + r) * 4;
        const float c0 = sp<float>(sm, PSM(cst_x))[(0 * kPMaxUnits + uu) * 16 + r];
        const float c1 = sp<float>(sm, PSM(cst_x))[(1 * kPMaxUnits + uu) * 16 + r];
        const float c2 = sp<float>(sm, PSM(cst_x))[(2 * kPMaxUnits + uu) * 16 + r];
        double pre = h2d(sp<uint16_t>(sm, PSM(convb_x))[uu * 16 + r]);
        pre = fma(h2d(cw[0]), double(c0), pre);
        pre = fma(h2d(cw[1]), double(c1), pre);
        pre = fma(h2d(cw[2]), double(c2), pre);
        pre = fma(h2d(cw[3]), xv, pre);
        const int ch = 16 * (w.u0 + uu) + r;
        float* gcs = L.conv_state;
        gcs[ch] = c1;
        gcs[C + ch] = c2;
        gcs[2 * C + ch] = float(xv);
        const double xc = silu_d(pre);
        yin[(xslot + uu) * 16 + r] = xc;
        if (diag) a.d_xc[ch] = xc;
      } else if (tid >= 64 && tid < 64 + w.nu * 16) {   // gate silu(z), in place of z
        const int rr = tid - 64;
        yin[(zslot + rr / 16) * 16 + rr % 16] = silu_d(yin[(zslot + rr / 16) * 16 + rr % 16]);
      } else if (tid >= 128 && tid < 128 + w.ns * 16) {   // own shared rows
        const int i = tid - 128;
        const int si = w.s0 + i / 16, r = i % 16;        // shared tile of the cluster, row in it
        double v = yin[(shslot + i / 16) * 16 + r];
        if (si < w.nbc) {                                 // a B/C row: conv step + SiLU
          const uint16_t* cw = sp<uint16_t>(sm, PSM(sh_convw)) + i * 4;
          const float* cst = sp<float>(sm, PSM(sh_cst));
          const float c0 = cst[i], c1 = cst[SHR + i], c2 = cst[2 * SHR + i];
          double pre = h2d(sp<uint16_t>(sm, PSM(sh_convb))[i]);
          pre = fma(h2d(cw[0]), double(c0), pre);
          pre = fma(h2d(cw[1]), double(c1), pre);
          pre = fma(h2d(cw[2]), double(c2), pre);
          pre = fma(h2d(cw[3]), v, pre);
          shst[i] = c1;
          shst[SHR + i] = c2;
          shst[2 * SHR + i] = float(v);
          v = silu_d(pre);
          if (diag) a.d_xc[E + 16 * si + r] = v;
          stg_c[i] = v;
        } else {                                          // a dt row: step size and decay of its head
          const int h = 16 * (w.cdt0 + si - w.nbc) + r;
          const double dt = softplus_d(v + double(sp<float>(sm, PSM(hd_dtb))[h]));
          const int o = 16 * w.nsbc + 32 * (si - w.s0 - w.nsbc) + r;   // dt tile: 16 steps, then 16 decays
          stg_c[o] = dt;
          stg_c[o + 16] = exp(dt * -exp(double(sp<float>(sm, PSM(hd_alog))[h])));
        }
        fence_async_smem();
      }
      // shared rows of the cluster: B/C rows (16 per tile), then per dt tile 16 steps
      // and 16 decays; this CTA's tiles are contiguous from shared row 16 s0 + 16 (s0 - nbc)+
      xsend(stg_c, shr + 16 * w.s0 + 16 * max(w.s0 - w.nbc, 0),
            unsigned((16 * w.nsbc + 32 * (w.ns - w.nsbc)) * 8), &xbars[EX_C], Q);
      if (!xwait(status, ctl, &xbars[EX_C], unsigned((2 * w.NS - w.nbc) * 16 * 8), par, 64u)) { alive = false; break; }
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
      // ---- G: own slice of the gated value and the sums of squares
      if (!tw_gather2(status, ctl, a.x_g + r0E, SE, reinterpret_cast<uint32_t*>(vs), a.x_gs, 2 * G, scratch32,
                      tag(l, XG), 64u)) {
        alive = false;
        break;
      }
      const double ssg = sum_partials(scratch32, G, redd);
      if (w.k == 0) {   // B/C conv state of this layer: every CTA has finished reading it
        for (int i = tid; i < w.nsbc * 16; i += kPThreads) {
          const int ch = E + 16 * w.s0 + i;
          for (int r = 0; r < 3; ++r) L.conv_state[size_t(r) * C + ch] = shst[r * SHR + i];
        }
      }
      if (!mbar_wait_compute(status, ctl, full_cd, par, 128u)) { alive = false; break; }
      // ---- A': gated RMSNorm on the slice -> the cluster
      const double rs_out = 1.0 / sqrt(ssg / double(E) + kEpsD);
      prep_slice(vs, sp<uint16_t>(sm, PSM(gnorm)), SE, rs_out, stg_a, redi, xs, cdiag ? a.d_x_out + r0E : nullptr,
                 cdiag ? a.d_xd_out + r0E : nullptr, E);
      xsend(stg_a, asm_a + w.r * BSE, unsigned(BSE), &xbars[EX_A_OUT], Q);
      if (!xwait(status, ctl, &xbars[EX_A_OUT], unsigned(Q * BSE), par, 128u)) { alive = false; break; }
      long long xsum_out;
      unsigned amax_out;
      slice_totals(asm_a, Q, SE, BSE, &xsum_out, &amax_out);
      const float am_out = half_to_float_bits(amax_out);
      const float sx_out = am_out > 0.f ? __fdiv_rn(am_out, 127.f) : 1.f;
      if (wdiag) {
        if (tid == 0) *a.d_sx_out = sx_out;
        plane_sums(asm_a, Q, SE, BSE, redi, a.d_xdsum_out);
      }
      // ---- B': codes and LoRA partials of the slice -> the cluster
      codes_and_lora_partials(xs, SE, sx_out, __frcp_rn(sx_out), am_out > 0.f, xqs, sp<int8_t>(sm, PSM(a_out)), R,
                              stg_b, cdiag ? a.d_xq_out + r0E : nullptr);
      if (R) xsend(stg_b, rcv_b + w.r * R, unsigned(4 * R), &xbars[EX_B_OUT], Q);
      // ---- out_proj scaffold on own tiles
      int nch_out = 1;
      if (w.no > 0) nch_out = scaffold_mma(sm + PSM(out_tiles), w.no, kg_out, asm_a, lgSE, BSE, part);
      if (R) {
        if (!xwait(status, ctl, &xbars[EX_B_OUT], unsigned(Q * 4 * R), par, 256u)) { alive = false; break; }
        lora_finish(rcv_b, Q, R, sp<uint16_t>(sm, PSM(sa_out)), sx_out, u, wdiag ? a.d_acc_out : nullptr, a.d_u_out);
        lora2_rows(sp<int8_t>(sm, PSM(out_bq)), w.no * 16, u, R, lo);
        csync();
      }
      // ---- R': residual rows and their sum of squares, published for the next layer
      const bool last = (l + 1 == a.n_layer);
      if (tid < w.no * 16) {
        const int o = w.o0 * 16 + tid;
        double y = h2d(sp<uint16_t>(sm, PSM(out_alpha))[tid]) * tile_row_value(part, tid / 16, nch_out, tid % 16, xsum_out);
        if (R) y = fma(h2d(sp<uint16_t>(sm, PSM(out_sb))[tid]), lo[tid], y);
        const float rn = float(double(resown[tid]) + y);
        resown[tid] = rn;
        if (!(last && a.layer_mode)) tw_put(a.x_r + o, __float_as_uint(rn), tag(l + 1, XR));
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
        if (lane == 0 && !(last && a.layer_mode)) tw_put_f64(a.x_rs + 2 * w.c, t, tag(l + 1, XR));
      }
      if (tid == 0) mbar_arrive(empty_cd);      // CD group consumed
    }

    // ---- LM head
    if (alive && !a.layer_mode) {
      const int L = a.n_layer;
      float* fres = sp<float>(sm, PSM(full)) + 2 * G;     // [D] residual, then [D] normalised
      float* xn = fres + D;
      if (tw_gather2(status, ctl, a.x_r, D, reinterpret_cast<uint32_t*>(fres), a.x_rs, 2 * G, scratch32, tag(L, XR),
                     512u)) {
        const double rs = 1.0 / sqrt(sum_partials(scratch32, G, redd) / double(D) + kEpsD);
        for (int k = tid; k < D; k += kPThreads) xn[k] = float((double(fres[k]) * rs) * h2d(a.normf_w[k]));
        csync();
        float best = -INFINITY;
        int besti = 0x7fffffff;
        float* hsum = sp<float>(sm, PSM(part));     // [2][CR][2]
        // warp 2 r + h takes half h of row r of every chunk; its lanes keep their
        // columns of the normalised residual in registers (kHV 8-column groups each)
        constexpr int kHV = 4;
        const int hrow = warp >> 1, hhalf = warp & 1;
        const int hn = D / 16, hb = hhalf * hn;      // 8-column groups per half row, first group of this half
        float xr[kHV][8];
#pragma unroll
        for (int m = 0; m < kHV; ++m)
#pragma unroll
          for (int e = 0; e < 8; ++e) xr[m][e] = lane + 32 * m < hn ? xn[(hb + lane + 32 * m) * 8 + e] : 0.f;
        for (int ci = 0; ci < head_chunks && alive; ++ci) {
          const int b = ci % NH;
          if (!mbar_wait_compute(status, ctl, full_h + b, unsigned(ci / NH) & 1u, 1024u)) { alive = false; break; }
          const int r0 = v0 + ci * CR, nr = min(CR, v1 - r0);
          float* hs = hsum + (ci & 1) * 2 * CR;
#pragma unroll
          for (int rsub = 0; rsub < CR / kHeadChunkRows; ++rsub) {
          const int row = hrow + kHeadChunkRows * rsub;
          if (row < nr) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            auto acc8 = [&](const float (&f)[8], const float* x) {
              acc[0] = fmaf(f[0], x[0], acc[0]); acc[1] = fmaf(f[1], x[1], acc[1]);
              acc[2] = fmaf(f[2], x[2], acc[2]); acc[3] = fmaf(f[3], x[3], acc[3]);
              acc[0] = fmaf(f[4], x[4], acc[0]); acc[1] = fmaf(f[5], x[5], acc[1]);
              acc[2] = fmaf(f[6], x[6], acc[2]); acc[3] = fmaf(f[7], x[7], acc[3]);
            };
            auto f16x8 = [](const uint4& wv, float (&f)[8]) {
              const __half2* wh = reinterpret_cast<const __half2*>(&wv);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 t2 = __half22float2(wh[i]);
                f[2 * i] = t2.x;
                f[2 * i + 1] = t2.y;
              }
            };
            const unsigned char* wrow = head_slot(b) + size_t(row) * head_row_bytes;
#pragma unroll
            for (int m = 0; m < kHV; ++m) {
              if (lane + 32 * m < hn) {
                float f[8];
                if (q8) i8x8_to_float(reinterpret_cast<const uint2*>(wrow)[hb + lane + 32 * m], f);
                else f16x8(reinterpret_cast<const uint4*>(wrow)[hb + lane + 32 * m], f);
                acc8(f, xr[m]);
              }
            }
            for (int c = lane + 32 * kHV; c < hn; c += 32) {   // half rows wider than kHV groups per lane
              float f[8];
              if (q8) i8x8_to_float(reinterpret_cast<const uint2*>(wrow)[hb + c], f);
              else f16x8(reinterpret_cast<const uint4*>(wrow)[hb + c], f);
              acc8(f, xn + (hb + c) * 8);
            }
            const float v = warp_sum((acc[0] + acc[1]) + (acc[2] + acc[3]));
            if (lane == 0) hs[row * 2 + hhalf] = v;
          }
          }
          csync();
          if (tid == 0) mbar_arrive(empty_h + b);      // the slot may be refilled
          if (tid < nr) {
            float lg = hs[tid * 2] + hs[tid * 2 + 1];
            if (q8) lg *= a.embed_s[r0 + tid];
            if (a.logits) a.logits[r0 + tid] = lg;
            if (lg > best || (lg == best && r0 + tid < besti)) { best = lg; besti = r0 + tid; }
          }
        }
        csync();
        // best over the threads that held rows
        if (tid < CR) {
          scratch32[2 * tid] = __float_as_uint(best);
          scratch32[2 * tid + 1] = uint32_t(besti);
        }
        csync();
        if (tid == 0) {
          float bv = -INFINITY;
          int bi = 0x7fffffff;
          for (int i = 0; i < CR; ++i) {
            const float v = __uint_as_float(scratch32[2 * i]);
            const int id = int(scratch32[2 * i + 1]);
            if (v > bv || (v == bv && id < bi)) { bv = v; bi = id; }
          }
          tw_put(a.x_head + 2 * w.c, __float_as_uint(bv), tag(L, XHEAD));
          tw_put(a.x_head + 2 * w.c + 1, uint32_t(bi), tag(L, XHEAD));
        }
        csync();
        if (w.c == 0 && alive) {
          if (tw_gather2(status, ctl, a.x_head, 2 * G, scratch32, a.x_head, 0, scratch32, tag(L, XHEAD), 2048u) &&
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
    }
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
