// Whole-token persistent decode kernel for batch 1 ("Density Field State Space
// Models", Section 4.1: the 48-layer forward of one decode token, here one launch).
//
// One CTA per SM for the whole token, warp-specialised:
//   * 16 compute warps run the layer's dependency chain;
//   * 1 producer warp streams each layer's per-CTA weight and state slices into
//     shared memory ahead of use: a few large bulk copies (cp.async.bulk, mbarrier
//     completion) for the tiles, plain 16-byte loads for the small per-row items.
//     Full/empty mbarrier pairs hand buffers between the two roles, so copy issue
//     never sits on the compute warps' critical path.
// Blocks exchange the few values a layer needs from one another through "tagged
// words": 64-bit words holding 32 data bits and a 32-bit tag (launch epoch, layer,
// exchange kind), stored and polled without fences -- a word is valid exactly
// when its tag matches.
//
// Per layer (B = 1):
//   R   all blocks gather the residual (d_model words) written by out_proj owners
//   -   every block recomputes x = fp16(rmsnorm(res) w), its int8 codes and digit planes
//   UIN blocks owning LoRA row j publish u_in[j] = A[j].xq * sA[j] * sx
//   -   exact int8 scaffold MMA on the block's in_proj tiles: z and x rows of its own
//       SSM rows, the dt tile of its heads and (a few blocks) one B/C tile, whose
//       scaffold values they publish (BC)
//   -   epilogue: + LoRA (needs UIN), conv step of its own x channels; every block
//       completes B and C itself (scaffold from BC + LoRA + conv)
//   G   SSM update of its own state rows, g = y silu(z) published as fp32
//   -   every block gathers g, recomputes the gated RMSNorm, codes and digit planes
//   UOUT blocks owning LoRA row j publish u_out[j]
//   R'  out_proj owners add their rows to the residual and publish it
// Final: gather the residual, final RMSNorm, stream this block's LM-head rows,
// publish (best logit, id); block 0 reduces to the greedy token.
//
// Every spin is bounded: a wait that gives up sets a status bit and an abort flag
// that makes every block leave the token early.
#pragma once

#include "common.cuh"

namespace dfssm {

constexpr int kMaxLayers = 64;
constexpr int kPThreads = 512;                    // compute threads
constexpr int kPWarps = kPThreads / 32;
constexpr int kPBlock = kPThreads + 32;           // + one producer warp
constexpr int kPMaxUnits = 2;                     // SSM row units (16 rows) per block
constexpr int kPMaxInTiles = 2 * kPMaxUnits + 3;  // z, x per unit + <= 2 dt tiles + <= 1 B/C tile
constexpr long long kSpinLimit = 1LL << 22;       // polls before a wait gives up (seconds)
constexpr int kHeadChunkRows = 8;

enum { XR = 0, XUIN = 1, XBC = 2, XG = 3, XUOUT = 4, XHEAD = 5 };

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
  int bc_bq, bc_sb, bc_convw, bc_convb, bc_cst, a_in, prenorm, sa_in, hd_dtb, hd_alog, hd_d, state;
  int ab_end;
  // layer group CD (refilled after out_proj)
  int out_tile, out_bq, out_alpha, out_sb, a_out, gnorm, sa_out;
  int cd_end;
  // working
  int res, gbuf, x16, digits, xq, part, yin, bcx, bcst_new, u_in, u_out, misc;
  int total;
};

struct __align__(16) PParams {
  // shape
  int n_layer, D, E, H, P, N, R, in_rows, C, vocab;
  int kg_in, kg_out;             // 256-column groups of the in/out projections
  int units, grid;               // SSM row units (E/16) and blocks
  int n_bc_tiles, dt_tile0;      // 2N/16 and first dt tile index
  int out_tiles;                 // D/16
  int layer_mode;                // 1: residual in/out from `residual`, no embedding / head
  PSmem sm;
  // io
  const uint16_t* embed; const uint16_t* normf_w; const int32_t* tok_in; int32_t* tok_out; float* logits;
  float* residual;               // layer mode: [D] in/out
  // workspace
  unsigned* status;              // status word
  unsigned* ctl;                 // [0] launch epoch, [1] abort flag
  unsigned long long* x_r;       // D residual words + one token word per block without an out_proj tile
  unsigned long long* x_g;       // E words
  unsigned long long* x_bc;      // 2N * 2 words
  unsigned long long* x_uin;     // R * 2 words
  unsigned long long* x_uout;    // R * 2 words
  unsigned long long* x_head;    // grid * 2 words
  // diagnostics of the last layer (workspace regions of dfssm_ws_layout)
  uint16_t* d_x_in; int8_t* d_xq_in; float* d_sx_in; int* d_acc_in; double* d_u_in; int8_t* d_xd_in;
  int* d_xdsum_in; double* d_zx; double* d_xc; float* d_g; uint16_t* d_x_out; int8_t* d_xq_out;
  float* d_sx_out; int* d_acc_out; double* d_u_out; int8_t* d_xd_out; int* d_xdsum_out; float* d_res;
  PLayer L[kMaxLayers];
};

// ------------------------------------------------------------------ primitives

DFSSM_DEV uint32_t smem_u32(const void* p) { return uint32_t(__cvta_generic_to_shared(p)); }

DFSSM_DEV void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
DFSSM_DEV void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
DFSSM_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}
DFSSM_DEV bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
DFSSM_DEV void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Named barrier 1 over the 16 compute warps only (the producer warp never joins).
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
DFSSM_DEV unsigned long long tw_load(const unsigned long long* p) {
  unsigned long long w;
  asm volatile("ld.volatile.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}
DFSSM_DEV void tw_put_f64(unsigned long long* p, double v, uint32_t tag) {
  const unsigned long long b = __double_as_longlong(v);
  tw_put(p, uint32_t(b), tag);
  tw_put(p + 1, uint32_t(b >> 32), tag);
}
DFSSM_DEV double f64_of(const uint32_t* w2) {
  return __longlong_as_double((static_cast<long long>(w2[1]) << 32) | w2[0]);
}

DFSSM_DEV bool aborted(const unsigned* ctl) { return *reinterpret_cast<volatile const unsigned*>(ctl + 1) != 0; }

DFSSM_DEV void give_up(unsigned* status, unsigned* ctl, unsigned bit) {
  atomicOr(status, bit);
  atomicExch(ctl + 1, 1u);
}

// Compute warps: gather n tagged words into dst (32-bit payloads).  Returns false
// (after flagging) if a word did not arrive within the spin limit.
DFSSM_DEV bool tw_gather(unsigned* status, unsigned* ctl, const unsigned long long* src, int n, uint32_t tag,
                         uint32_t* dst, unsigned bit) {
  bool ok = true;
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
        if (pending & (1u << i)) w[i] = tw_load(src + idx[i]);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if ((pending & (1u << i)) && uint32_t(w[i] >> 32) == tag) {
          dst[idx[i]] = uint32_t(w[i]);
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

// Compute-warp reductions (fixed order, identical in every block).
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
DFSSM_DEV float cmax_f(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  if (lane == 0) red[warp] = v;
  csync();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kPWarps; ++w) t = fmaxf(t, red[w]);
  csync();
  return t;
}

// ------------------------------------------------------------------ assignment

struct PWork {
  int c;                 // block index
  int u0, nu;            // SSM units [u0, u0 + nu)
  int h0, h1;            // heads touched [h0, h1]
  int ndt;               // dt tiles (1 or 2)
  int bc_index;          // which B/C tile this block owns, or -1
  int ntile;             // in_proj tiles: nu z tiles, nu x tiles, ndt dt tiles, [B/C tile]
  int out_tile;          // out_proj tile or -1
};

DFSSM_DEV PWork assign(const PParams& a) {
  PWork w;
  const int c = blockIdx.x, G = a.grid;
  w.c = c;
  const int base = a.units / G, extra = a.units % G;
  w.u0 = c * base + min(c, extra);
  w.nu = base + (c < extra ? 1 : 0);
  w.h0 = (16 * w.u0) / a.P;
  w.h1 = (16 * (w.u0 + w.nu) - 1) / a.P;
  w.ndt = w.h1 / 16 - w.h0 / 16 + 1;
  w.bc_index = (G - 1 - c < a.n_bc_tiles) ? G - 1 - c : -1;
  w.ntile = 2 * w.nu + w.ndt + (w.bc_index >= 0 ? 1 : 0);
  w.out_tile = c < a.out_tiles ? c : -1;
  return w;
}

// The four contiguous tile ranges of a block's in_proj rows: (first tile, count).
DFSSM_DEV void tile_range(const PParams& a, const PWork& w, int k, int* t0, int* n) {
  switch (k) {
    case 0: *t0 = w.u0; *n = w.nu; break;                                   // z rows
    case 1: *t0 = a.E / 16 + w.u0; *n = w.nu; break;                        // x rows
    case 2: *t0 = a.dt_tile0 + w.h0 / 16; *n = w.ndt; break;                // dt rows
    default: *t0 = 2 * a.E / 16 + max(w.bc_index, 0); *n = w.bc_index >= 0 ? 1 : 0; break;  // B/C rows
  }
}

// in_proj tile index of tile slot ti (slots ordered z, x, dt, B/C)
DFSSM_DEV int slot_tile(const PParams& a, const PWork& w, int ti) {
  int t0, n;
  for (int k = 0; k < 4; ++k) {
    tile_range(a, w, k, &t0, &n);
    if (ti < n) return t0 + ti;
    ti -= n;
  }
  return -1;
}

DFSSM_DEV int first_lora_row(const PParams& a) { return a.grid - 1 - int(blockIdx.x); }

template <typename T>
DFSSM_DEV T* sp(unsigned char* sm, int off) { return reinterpret_cast<T*>(sm + off); }

// ------------------------------------------------------------------ producer

// Copy `bytes` (multiple of 16) with the producer warp's asynchronous 16-byte copies
// (cp.async); each lane later hands their completion to the group's mbarrier.
DFSSM_DEV void warp_copy(unsigned char* dst, const void* src, int bytes) {
  const unsigned char* s = static_cast<const unsigned char*>(src);
  for (int i = int(threadIdx.x & 31); i < bytes / 16; i += 32)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(smem_u32(dst + 16 * i)), "l"(s + 16 * i)
                 : "memory");
}
// Every producer lane: arrive on `bar` once all of its earlier cp.async copies land.
DFSSM_DEV void warp_copies_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
}

// Producer warp: the AB group of layer l.  Lane 0 arms `full` with the bulk bytes
// and issues the bulk copies; all lanes copy the small items asynchronously and
// arrive on `full` when their copies land (arrival count 1 + 32).
DFSSM_DEV void produce_ab(const PParams& a, const PWork& w, const PLayer& L, unsigned char* sm, uint64_t* full) {
  const PSmem& s = a.sm;
  const int lane = threadIdx.x & 31;
  const unsigned tile_bytes = unsigned(a.kg_in) * 512u;
  if (lane == 0) {
    unsigned bytes = unsigned(w.ntile) * tile_bytes + 2u * a.D + unsigned(w.nu) * 16u * a.N * 4u;
    if (a.R) bytes += unsigned(w.ntile) * 16u * a.R + 2u * a.N * a.R + unsigned(a.D);
    mbar_expect_tx(full, bytes);
    int slot = 0;
    for (int k = 0; k < 4; ++k) {
      int t0, n;
      tile_range(a, w, k, &t0, &n);
      if (n == 0) continue;
      bulk_g2s(sm + s.in_tiles + slot * tile_bytes, L.in_bits + size_t(t0) * a.kg_in * 128, n * tile_bytes, full);
      if (a.R) bulk_g2s(sm + s.in_bq + slot * 16 * a.R, L.in_B + size_t(t0) * 16 * a.R, n * 16u * a.R, full);
      slot += n;
    }
    if (a.R) {
      bulk_g2s(sm + s.bc_bq, L.in_B + size_t(2 * a.E) * a.R, 2u * a.N * a.R, full);
      const int j = first_lora_row(a);
      bulk_g2s(sm + s.a_in, L.in_A + size_t(j < a.R ? j : 0) * a.D, unsigned(a.D), full);
    }
    bulk_g2s(sm + s.prenorm, L.prenorm_w, 2u * a.D, full);
    bulk_g2s(sm + s.state, L.ssm_state + size_t(16 * w.u0) * a.N, unsigned(w.nu) * 16u * a.N * 4u, full);
  }
  int slot = 0;
  for (int k = 0; k < 4; ++k) {
    int t0, n;
    tile_range(a, w, k, &t0, &n);
    if (n == 0) continue;
    warp_copy(sm + s.in_alpha + slot * 32, L.in_alpha + size_t(t0) * 16, n * 32);
    warp_copy(sm + s.in_sb + slot * 32, (L.in_sB ? L.in_sB : L.in_alpha) + size_t(t0) * 16, n * 32);
    slot += n;
  }
  const int ch = 16 * w.u0;
  warp_copy(sm + s.convw_x, L.conv_w + size_t(ch) * 4, w.nu * 128);
  warp_copy(sm + s.convb_x, L.conv_b + ch, w.nu * 32);
  for (int r = 0; r < 3; ++r)
    warp_copy(sm + s.cst_x + r * kPMaxUnits * 64, L.conv_state + size_t(r) * a.C + ch, w.nu * 64);
  const int bc0 = 2 * a.E;
  warp_copy(sm + s.bc_sb, (L.in_sB ? L.in_sB : L.in_alpha) + bc0, 4 * a.N);
  warp_copy(sm + s.bc_convw, L.conv_w + size_t(a.E) * 4, 16 * a.N);
  warp_copy(sm + s.bc_convb, L.conv_b + a.E, 4 * a.N);
  for (int r = 0; r < 3; ++r) warp_copy(sm + s.bc_cst + r * 8 * a.N, L.conv_state + size_t(r) * a.C + a.E, 8 * a.N);
  if (a.R) warp_copy(sm + s.sa_in, L.in_sA, 2 * a.R);
  warp_copy(sm + s.hd_dtb, L.dt_bias, 4 * a.H);
  warp_copy(sm + s.hd_alog, L.A_log, 4 * a.H);
  warp_copy(sm + s.hd_d, L.D, 4 * a.H);
  warp_copies_arrive(full);
}

DFSSM_DEV void produce_cd(const PParams& a, const PWork& w, const PLayer& L, unsigned char* sm, uint64_t* full) {
  const PSmem& s = a.sm;
  const int lane = threadIdx.x & 31;
  const unsigned tile_bytes = unsigned(a.kg_out) * 512u;
  if (lane == 0) {
    unsigned bytes = 2u * a.E;
    if (w.out_tile >= 0) bytes += tile_bytes + (a.R ? 16u * a.R : 0u);
    if (a.R) bytes += unsigned(a.E);
    mbar_expect_tx(full, bytes);
    bulk_g2s(sm + s.gnorm, L.gnorm_w, 2u * a.E, full);
    if (w.out_tile >= 0) {
      bulk_g2s(sm + s.out_tile, L.out_bits + size_t(w.out_tile) * a.kg_out * 128, tile_bytes, full);
      if (a.R) bulk_g2s(sm + s.out_bq, L.out_B + size_t(w.out_tile) * 16 * a.R, 16u * a.R, full);
    }
    if (a.R) {
      const int j = first_lora_row(a);
      bulk_g2s(sm + s.a_out, L.out_A + size_t(j < a.R ? j : 0) * a.E, unsigned(a.E), full);
    }
  }
  if (w.out_tile >= 0) {
    warp_copy(sm + s.out_alpha, L.out_alpha + size_t(w.out_tile) * 16, 32);
    warp_copy(sm + s.out_sb, (L.out_sB ? L.out_sB : L.out_alpha) + size_t(w.out_tile) * 16, 32);
  }
  if (a.R) warp_copy(sm + s.sa_out, L.out_sA, 2 * a.R);
  warp_copies_arrive(full);
}

// ------------------------------------------------------------------ activation prep

// Exact fp16 -> fp32 by bit construction for normal values (no convert
// instruction); zero, subnormal and non-finite values take the hardware path.
DFSSM_DEV float half_to_float_bits(uint32_t h) {
  const uint32_t e = (h >> 10) & 0x1fu;
  if (e == 0u || e == 31u) return h2f(uint16_t(h));
  return __uint_as_float(((h & 0x8000u) << 16) | ((e + 112u) << 23) | ((h & 0x3ffu) << 13));
}

// x * 2^24 as an integer, exact for every finite fp16 (|result| < 2^40 fits int64;
// the packed-digit path only calls it when |x| <= 127, where it fits int32).
DFSSM_DEV int half_times_2p24(uint32_t h) {
  const uint32_t e = (h >> 10) & 0x1fu, m = h & 0x3ffu;
  const int X = e == 0u ? int(m) : int((m | 0x400u) << (e - 1u));
  return (h & 0x8000u) ? -X : X;
}

// fp16 bits of z = (v * rs) * w, correctly rounded from the fp64 product.  The
// fp32 product lies within 4 fp32 ulps of it; if its low 13 mantissa bits are more
// than 4 away from the fp16 rounding midpoint (0x1000) and z is in the fp16 normal
// range, rounding the fp32 value is already the answer (done here with integer
// ops); otherwise fp64 decides.
DFSSM_DEV uint16_t norm_fp16(float v, double rs, float rs32, float wf) {
  const float z = (v * rs32) * wf;
  const uint32_t bits = __float_as_uint(z);
  const uint32_t ez = (bits >> 23) & 0xffu;
  const int low13 = int(bits & 0x1fffu);
  if (ez >= 113u && ez <= 141u && abs(low13 - 0x1000) > 4) {
    uint32_t hm = ((ez - 112u) << 10) | ((bits >> 13) & 0x3ffu);
    hm += low13 > 0x1000 ? 1u : 0u;
    return uint16_t(hm | ((bits >> 16) & 0x8000u));
  }
  return d2h((double(v) * rs) * double(wf));
}

// Round-to-nearest-even of |t| < 2^22 via the 1.5 * 2^23 add (no convert instruction).
DFSSM_DEV int rint_small(float t, float* r) {
  const float m = t + 12582912.0f;
  *r = m - 12582912.0f;
  return __float_as_int(m) - 0x4B400000;
}

// Same decision as quant_code: clamp(rint(x / sx), -127, 127) with the fp32 IEEE
// divide; the product x * rcp is within 3 * 2^-24 |x/sx| of the correctly rounded
// quotient, so the divide is only needed near a half-integer.
DFSSM_DEV int quant_code_bits(float x, float sx, float rcp) {
  const float t = x * rcp;
  float r;
  int q = rint_small(t, &r);
  if (fabsf(fabsf(t - r) - 0.5f) <= 4.0e-5f) q = __float2int_rn(__fdiv_rn(x, sx));
  return max(-127, min(127, q));
}

// Four consecutive fp16 values -> their packed balanced base-256 digit bytes, one
// 32-bit word per digit plane (byte e = element e); |x| <= 127 (4 planes).
DFSSM_DEV void pack_digits4(const uint32_t (&h)[4], uint32_t (&planes)[4]) {
  uint32_t P[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) P[e] = (uint32_t(half_times_2p24(h[e])) + 0x80808080u) ^ 0x80808080u;
  const uint32_t t01 = __byte_perm(P[0], P[1], 0x5140), t23 = __byte_perm(P[2], P[3], 0x5140);
  const uint32_t u01 = __byte_perm(P[0], P[1], 0x7362), u23 = __byte_perm(P[2], P[3], 0x7362);
  planes[0] = __byte_perm(t01, t23, 0x5410);
  planes[1] = __byte_perm(t01, t23, 0x7632);
  planes[2] = __byte_perm(u01, u23, 0x5410);
  planes[3] = __byte_perm(u01, u23, 0x7632);
}

// x = fp16((v * rs) * w) for K values (fp32 src in smem), rs = 1/sqrt(mean(v^2)+eps)
// in fp64, and its scaffold digit planes (stride K+16) with their sums in tsum[6].
// Blocks that own a LoRA row (`codes`) also take the fp32 LoRA decision: amax, sx
// and int8 codes.  Four consecutive elements per thread per step.  Returns sx
// (1 when `codes` is false).
DFSSM_DEV float prep_activation(const float* v, const uint16_t* w, int K, bool codes, uint16_t* x16, int8_t* xq,
                                int8_t* dg, int* tsum, double* redd, float* redf, int* redi, uint16_t* x_diag,
                                int8_t* xq_diag, int8_t* xd_diag, int* xdsum_diag, float* sx_diag) {
  const int tid = threadIdx.x, K4 = K / 4, DS = K + 16;
  const bool keep = codes || x_diag;
  double ss = 0.0;
  for (int i = tid; i < K4; i += kPThreads) {
    const float4 f = reinterpret_cast<const float4*>(v)[i];
    ss = fma(double(f.x), double(f.x), ss);
    ss = fma(double(f.y), double(f.y), ss);
    ss = fma(double(f.z), double(f.z), ss);
    ss = fma(double(f.w), double(f.w), ss);
  }
  ss = csum_d(ss, redd);
  const double rs = 1.0 / sqrt(ss / double(K) + kEpsD);
  const float rs32 = float(rs);
  uint32_t am_bits = 0;                   // max |x| as fp16 bits (monotone for non-negative values)
  uint32_t big = 0;                       // any |x| > 127: the digit planes need the 6-plane path
  int ts[kDigits] = {0, 0, 0, 0, 0, 0};
  for (int i = tid; i < K4; i += kPThreads) {
    const float4 f = reinterpret_cast<const float4*>(v)[i];
    const uint2 wv = reinterpret_cast<const uint2*>(w)[i];
    uint32_t h[4];
    h[0] = norm_fp16(f.x, rs, rs32, half_to_float_bits(wv.x & 0xffffu));
    h[1] = norm_fp16(f.y, rs, rs32, half_to_float_bits(wv.x >> 16));
    h[2] = norm_fp16(f.z, rs, rs32, half_to_float_bits(wv.y & 0xffffu));
    h[3] = norm_fp16(f.w, rs, rs32, half_to_float_bits(wv.y >> 16));
    const uint32_t m4 = max(max(h[0] & 0x7fffu, h[1] & 0x7fffu), max(h[2] & 0x7fffu, h[3] & 0x7fffu));
    am_bits = max(am_bits, m4);
    if (keep) reinterpret_cast<uint2*>(x16)[i] = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
    uint32_t planes[kDigits];
    if (m4 <= 0x57f0u) {                  // every |x| <= 127: four packed digit planes
      uint32_t p4[4];
      pack_digits4(h, p4);
#pragma unroll
      for (int d = 0; d < 4; ++d) planes[d] = p4[d];
      planes[4] = planes[5] = 0u;
    } else {
      big = 1u;
#pragma unroll
      for (int d = 0; d < kDigits; ++d) planes[d] = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int8_t d6[kDigits];
        fp16_digits(uint16_t(h[e]), d6);
#pragma unroll
        for (int d = 0; d < kDigits; ++d) planes[d] |= (uint32_t(uint8_t(d6[d]))) << (8 * e);
      }
    }
#pragma unroll
    for (int d = 0; d < kDigits; ++d) {
      *reinterpret_cast<uint32_t*>(dg + d * DS + 4 * i) = planes[d];
      ts[d] = __dp4a(int(planes[d]), 0x01010101, ts[d]);
    }
    if (x_diag) {
      reinterpret_cast<uint2*>(x_diag)[i] = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
#pragma unroll
      for (int d = 0; d < kDigits; ++d) reinterpret_cast<uint32_t*>(xd_diag + size_t(d) * K)[i] = planes[d];
    }
  }
  (void)big;
#pragma unroll
  for (int d = 0; d < kDigits; ++d) ts[d] = warp_sum_i(ts[d]);
  const int lane = tid & 31, warp = tid >> 5;
  if (lane == 0) {
#pragma unroll
    for (int d = 0; d < kDigits; ++d) redi[d * kPWarps + warp] = ts[d];
  }
  float sx = 1.f;
  if (codes) {
    const float am = cmax_f(half_to_float_bits(am_bits), redf);   // (also orders the redi writes)
    sx = am > 0.f ? __fdiv_rn(am, 127.f) : 1.f;
    const float rcp = __frcp_rn(sx);
    for (int i = tid; i < K4; i += kPThreads) {
      const uint2 hv = reinterpret_cast<const uint2*>(x16)[i];
      const uint32_t hh[4] = {hv.x & 0xffffu, hv.x >> 16, hv.y & 0xffffu, hv.y >> 16};
      uint32_t qw = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = am > 0.f ? quant_code_bits(half_to_float_bits(hh[e]), sx, rcp) : 0;
        qw |= (uint32_t(q) & 0xffu) << (8 * e);
      }
      reinterpret_cast<uint32_t*>(xq)[i] = qw;
      if (xq_diag) reinterpret_cast<uint32_t*>(xq_diag)[i] = qw;
    }
  } else {
    csync();
  }
  if (tid < kDigits) {
    int t = 0;
#pragma unroll
    for (int ww = 0; ww < kPWarps; ++ww) t += redi[tid * kPWarps + ww];
    tsum[tid] = t;
    if (xdsum_diag) xdsum_diag[tid] = t;
  }
  if (sx_diag && tid == 0) *sx_diag = sx;
  csync();
  return sx;
}

// One LoRA stage-1 row per warp: acc = A[j] . xq (exact), u = acc * sA[j] * sx.
DFSSM_DEV void lora_row(const int8_t* Arow, const int8_t* xq, int K, float sx, uint16_t sA, int* acc_out,
                        double* u_out) {
  const int lane = threadIdx.x & 31;
  const int* A4 = reinterpret_cast<const int*>(Arow);
  const int* q4 = reinterpret_cast<const int*>(xq);
  int acc = 0;
  for (int i = lane; i < K / 4; i += 32) acc = __dp4a(A4[i], q4[i], acc);
  acc = warp_sum_i(acc);
  *acc_out = acc;
  *u_out = (double(acc) * h2d(sA)) * double(sx);
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
// (tile, kgroup chunk); int32 partials to part[unit][16][kDigits].  Four
// independent accumulator sets (one per 64-column subtile) keep the tensor pipe
// busy instead of one serial MMA chain.  Returns the chunks per tile.
DFSSM_DEV int scaffold_mma(const unsigned char* tiles, int ntile, int kg, const int8_t* dg, int K, int* part) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  int nchunk = kPWarps / ntile;
  if (nchunk < 1) nchunk = 1;
  if (nchunk > kg) nchunk = kg;
  const int DS = K + 16;
  const int nunits = ntile * nchunk;
  const int8_t* drow = dg + (g < kDigits ? g : 0) * DS + 4 * t;
  for (int unit = warp; unit < nunits; unit += kPWarps) {
    const int ti = unit / nchunk, ci = unit % nchunk;
    const int kg_lo = ci * kg / nchunk, kg_hi = (ci + 1) * kg / nchunk;
    int acc[4][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}, {0, 0, 0, 0}, {0, 0, 0, 0}};
    const uint4* tw = reinterpret_cast<const uint4*>(tiles + size_t(ti) * kg * 512);
    for (int kgi = kg_lo; kgi < kg_hi; ++kgi) {
      const uint4 wv = tw[kgi * 32 + lane];
      const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
          uint32_t af[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) af[q] = sign_bytes(words[kt], 4 * ch + q);
          const int k0 = kgi * kTileCols + kt * 64 + ch * 32;
          uint32_t b0 = 0, b1 = 0;
          if (g < kDigits) {
            b0 = *reinterpret_cast<const uint32_t*>(drow + k0);
            b1 = *reinterpret_cast<const uint32_t*>(drow + k0 + 16);
          }
          mma_s8_16832(acc[kt], af, b0, b1);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[0][i] += acc[1][i] + acc[2][i] + acc[3][i];
    int* p = part + unit * 16 * kDigits;
    if (2 * t < kDigits) {
      p[g * kDigits + 2 * t] = acc[0][0];
      p[(g + 8) * kDigits + 2 * t] = acc[0][2];
    }
    if (2 * t + 1 < kDigits) {
      p[g * kDigits + 2 * t + 1] = acc[0][1];
      p[(g + 8) * kDigits + 2 * t + 1] = acc[0][3];
    }
  }
  csync();
  return nchunk;
}

// Scaffold value (without alpha) of row r of tile ti from the unit partials.
DFSSM_DEV double tile_row_value(const int* part, int ti, int nchunk, int r, const int* T) {
  int q[kDigits];
#pragma unroll
  for (int d = 0; d < kDigits; ++d) {
    int s = 0;
    for (int c = 0; c < nchunk; ++c) s += part[((ti * nchunk + c) * 16 + r) * kDigits + d];
    q[d] = s;
  }
  return scaffold_value(q, T);
}

// ------------------------------------------------------------------ the kernel

__global__ void __launch_bounds__(kPBlock, 1) k_decode_persistent(const __grid_constant__ PParams pa) {
  extern __shared__ __align__(128) unsigned char sm[];
  // The parameter block (~11 KB, mostly the per-layer pointer table) is read with
  // runtime layer indices all through the token; a shared-memory copy keeps those
  // reads off the small constant cache.
  __shared__ __align__(16) unsigned char pbuf[sizeof(PParams)];
  __shared__ __align__(8) uint64_t bars[8];   // full AB, empty AB, full CD, empty CD, full head x2, empty head x2
  __shared__ double redd[kPWarps];
  __shared__ float redf[kPWarps];
  __shared__ int redi[kDigits * kPWarps];
  __shared__ int tsum[kDigits];
  __shared__ double dt_h[4];
  __shared__ double dA_h[4];
  for (int i = threadIdx.x; i < int(sizeof(PParams) / 16); i += blockDim.x)
    reinterpret_cast<uint4*>(pbuf)[i] = reinterpret_cast<const uint4*>(&pa)[i];
  const PParams& a = *reinterpret_cast<const PParams*>(pbuf);
  uint64_t* full_ab = &bars[0];
  uint64_t* empty_ab = &bars[1];
  uint64_t* full_cd = &bars[2];
  uint64_t* empty_cd = &bars[3];
  uint64_t* full_h = &bars[4];
  uint64_t* empty_h = &bars[6];
  if (threadIdx.x == 0) {
    mbar_init(full_ab, 1 + 32);
    mbar_init(empty_ab, 1);
    mbar_init(full_cd, 1 + 32);
    mbar_init(empty_cd, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(full_h + i, 1);
      mbar_init(empty_h + i, 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();   // the only barrier the producer warp joins

  const PSmem& s = a.sm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const PWork w = assign(a);
  const int G = a.grid;
  const int v0 = int((long long)w.c * a.vocab / G), v1 = int((long long)(w.c + 1) * a.vocab / G);
  const int head_chunks = (v1 - v0 + kHeadChunkRows - 1) / kHeadChunkRows;
  const unsigned head_row_bytes = 2u * a.D;

  // ================================================================ producer warp
  if (warp == kPWarps) {
    bool ok = true;
    unsigned ab_issued = 0, cd_issued = 0, h_issued[2] = {0, 0};
    for (int l = 0; l < a.n_layer && ok; ++l) {
      if (l > 0 && lane == 0) ok = mbar_wait(a.status, a.ctl, empty_ab, unsigned(l - 1) & 1u, 4096u);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      produce_ab(a, w, a.L[l], sm, full_ab);
      ++ab_issued;
      if (l > 0 && lane == 0) ok = mbar_wait(a.status, a.ctl, empty_cd, unsigned(l - 1) & 1u, 8192u);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      produce_cd(a, w, a.L[l], sm, full_cd);
      ++cd_issued;
    }
    if (ok && !a.layer_mode) {
      // the LM-head ring reuses the AB group once the last layer's SSM is done
      if (lane == 0) ok = mbar_wait(a.status, a.ctl, empty_ab, unsigned(a.n_layer - 1) & 1u, 4096u);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      for (int ci = 0; ci < head_chunks && ok; ++ci) {
        const int b = ci & 1;
        if (lane == 0) {
          if (ci >= 2) ok = mbar_wait(a.status, a.ctl, empty_h + b, unsigned((ci >> 1) - 1) & 1u, 16384u);
          if (ok) {
            const int r0 = v0 + ci * kHeadChunkRows, nr = min(kHeadChunkRows, v1 - r0);
            mbar_expect_tx(full_h + b, nr * head_row_bytes);
            bulk_g2s(sm + size_t(b) * kHeadChunkRows * head_row_bytes, a.embed + size_t(r0) * a.D,
                     nr * head_row_bytes, full_h + b);
            ++h_issued[b];
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
    }
    // let every issued copy land before leaving (the block's shared memory stays
    // alive until all its threads exit)
    if (lane == 0) {
      long long spins = 0;
      if (ab_issued) while (!mbar_try_wait(full_ab, (ab_issued - 1) & 1u) && ++spins < kSpinLimit) {}
      if (cd_issued) while (!mbar_try_wait(full_cd, (cd_issued - 1) & 1u) && ++spins < kSpinLimit) {}
      for (int b = 0; b < 2; ++b)
        if (h_issued[b]) while (!mbar_try_wait(full_h + b, (h_issued[b] - 1) & 1u) && ++spins < kSpinLimit) {}
    }
    return;
  }

  // ================================================================ compute warps
  const uint32_t tagbase = *reinterpret_cast<volatile const unsigned*>(a.ctl) << 16;   // launch epoch
  auto tag = [&](int l, int kind) { return tagbase + uint32_t(l * 8 + kind + 1); };
  unsigned* status = a.status;
  unsigned* ctl = a.ctl;

  float* res = sp<float>(sm, s.res);
  float* gbuf = sp<float>(sm, s.gbuf);
  uint16_t* x16 = sp<uint16_t>(sm, s.x16);
  int8_t* dg = sp<int8_t>(sm, s.digits);
  int8_t* xq = sp<int8_t>(sm, s.xq);
  int* part = sp<int>(sm, s.part);
  double* yin = sp<double>(sm, s.yin);      // [kPMaxInTiles * 16] in_proj outputs of own tiles (slot order)
  double* bcx = sp<double>(sm, s.bcx);      // [2N] B/C after conv
  float* bcst_new = sp<float>(sm, s.bcst_new);
  double* u_in = sp<double>(sm, s.u_in);
  double* u_out = sp<double>(sm, s.u_out);
  uint32_t* scratch32 = sp<uint32_t>(sm, s.misc);
  double* lo = reinterpret_cast<double*>(gbuf);   // LoRA stage-2 sums (the gated buffer is free then)
  const int zslot = 0, xslot = w.nu, dtslot = 2 * w.nu, bcslot = 2 * w.nu + w.ndt;

  // ---- layer-0 residual
  if (a.layer_mode) {
    for (int k = tid; k < a.D; k += kPThreads) res[k] = a.residual[k];
  } else {
    int t = a.tok_in[0];
    if (t < 0 || t >= a.vocab) {
      if (tid == 0) atomicOr(status, 2u);
      t = t < 0 ? 0 : a.vocab - 1;
    }
    for (int k = tid; k < a.D; k += kPThreads) res[k] = h2f(a.embed[size_t(t) * a.D + k]);
  }
  csync();

  bool alive = true;
  for (int l = 0; l < a.n_layer && alive; ++l) {
    const PLayer& L = a.L[l];
    const bool diag = (l == a.n_layer - 1);
    const unsigned par = unsigned(l) & 1u;

    // ---- R: residual entering this layer
    if (l > 0) {
      if (!tw_gather(status, ctl, a.x_r, a.D + G - a.out_tiles, tag(l, XR), reinterpret_cast<uint32_t*>(res), 4u)) {
        alive = false;
        break;
      }
    }
    if (!mbar_wait_compute(status, ctl, full_ab, par, 8u)) { alive = false; break; }

    // ---- pre-norm, codes, digit planes
    const bool wdiag = diag && w.c == 0;
    const bool lora_block = a.R && first_lora_row(a) < a.R;
    const float sx_in = prep_activation(res, sp<uint16_t>(sm, s.prenorm), a.D, lora_block || wdiag, x16, xq, dg, tsum,
                                        redd, redf, redi,
                                        wdiag ? a.d_x_in : nullptr, wdiag ? a.d_xq_in : nullptr,
                                        wdiag ? a.d_xd_in : nullptr, wdiag ? a.d_xdsum_in : nullptr,
                                        wdiag ? a.d_sx_in : nullptr);
    // ---- UIN: this block's LoRA row
    if (a.R && warp == 0) {
      const int j = first_lora_row(a);
      if (j < a.R) {
        int acc;
        double u;
        lora_row(sp<int8_t>(sm, s.a_in), xq, a.D, sx_in, sp<uint16_t>(sm, s.sa_in)[j], &acc, &u);
        if (lane == 0) {
          tw_put_f64(a.x_uin + 2 * j, u, tag(l, XUIN));
          if (diag) { a.d_acc_in[j] = acc; a.d_u_in[j] = u; }
        }
      }
    }
    // ---- in_proj scaffold on own tiles
    const int nch_in = scaffold_mma(sm + s.in_tiles, w.ntile, a.kg_in, dg, a.D, part);
    if (tid < w.ntile * 16) {
      const int ti = tid / 16, r = tid % 16;
      const double v = h2d(sp<uint16_t>(sm, s.in_alpha)[tid]) * tile_row_value(part, ti, nch_in, r, tsum);
      yin[tid] = v;
      if (ti == bcslot) tw_put_f64(a.x_bc + 2 * (16 * w.bc_index + r), v, tag(l, XBC));
    }
    // ---- u_in, LoRA stage 2 of own rows
    if (a.R) {
      if (!tw_gather(status, ctl, a.x_uin, 2 * a.R, tag(l, XUIN), scratch32, 16u)) { alive = false; break; }
      if (tid < a.R) u_in[tid] = f64_of(scratch32 + 2 * tid);
      csync();
      lora2_rows(sp<int8_t>(sm, s.in_bq), w.ntile * 16, u_in, a.R, lo);
      csync();
    }
    // ---- epilogue of own rows
    if (tid < w.ntile * 16) {
      const int ti = tid / 16;
      double y = yin[tid];
      if (a.R) y = fma(h2d(sp<uint16_t>(sm, s.in_sb)[tid]), lo[tid], y);
      yin[tid] = y;
      if (diag) {
        const int row = slot_tile(a, w, ti) * 16 + tid % 16;
        const int h = row - (2 * a.E + 2 * a.N);
        if (row < a.in_rows && (ti < dtslot || ti == bcslot || (h >= w.h0 && h <= w.h1))) a.d_zx[row] = y;
      }
    }
    csync();
    if (tid < w.nu * 16) {                 // conv step of own x channels, in place
      const int u = tid / 16, r = tid % 16;
      const double xv = yin[(xslot + u) * 16 + r];
      const uint16_t* cw = sp<uint16_t>(sm, s.convw_x) + (u * 16 + r) * 4;
      const float c0 = sp<float>(sm, s.cst_x)[(0 * kPMaxUnits + u) * 16 + r];
      const float c1 = sp<float>(sm, s.cst_x)[(1 * kPMaxUnits + u) * 16 + r];
      const float c2 = sp<float>(sm, s.cst_x)[(2 * kPMaxUnits + u) * 16 + r];
      double pre = h2d(sp<uint16_t>(sm, s.convb_x)[u * 16 + r]);
      pre = fma(h2d(cw[0]), double(c0), pre);
      pre = fma(h2d(cw[1]), double(c1), pre);
      pre = fma(h2d(cw[2]), double(c2), pre);
      pre = fma(h2d(cw[3]), xv, pre);
      const int ch = 16 * (w.u0 + u) + r;
      float* gcs = L.conv_state;
      gcs[ch] = c1;
      gcs[a.C + ch] = c2;
      gcs[2 * a.C + ch] = float(xv);
      const double xc = silu_d(pre);
      yin[(xslot + u) * 16 + r] = xc;
      if (diag) a.d_xc[ch] = xc;
    } else if (tid >= 32 && tid < 32 + w.nu * 16) {   // gate silu(z), in place of z
      const int rr = tid - 32;
      yin[(zslot + rr / 16) * 16 + rr % 16] = silu_d(yin[(zslot + rr / 16) * 16 + rr % 16]);
    } else if (tid >= 64 && tid <= 64 + (w.h1 - w.h0)) {   // per-head step size and decay
      const int hi = tid - 64, h = w.h0 + hi;
      const double dt = softplus_d(yin[(dtslot + (h / 16 - w.h0 / 16)) * 16 + (h % 16)] +
                                   double(sp<float>(sm, s.hd_dtb)[h]));
      dt_h[hi] = dt;
      dA_h[hi] = exp(dt * -exp(double(sp<float>(sm, s.hd_alog)[h])));
    }
    // ---- B and C: gathered scaffold + LoRA + conv (every block), new state kept by block 0
    if (!tw_gather(status, ctl, a.x_bc, 4 * a.N, tag(l, XBC), scratch32, 32u)) { alive = false; break; }
    if (a.R) {
      lora2_rows(sp<int8_t>(sm, s.bc_bq), 2 * a.N, u_in, a.R, lo);
      csync();
    }
    for (int i = tid; i < 2 * a.N; i += kPThreads) {
      double y = f64_of(scratch32 + 2 * i);
      if (a.R) y = fma(h2d(sp<uint16_t>(sm, s.bc_sb)[i]), lo[i], y);
      const uint16_t* cw = sp<uint16_t>(sm, s.bc_convw) + i * 4;
      const float* cst = sp<float>(sm, s.bc_cst);
      const float c0 = cst[i], c1 = cst[2 * a.N + i], c2 = cst[4 * a.N + i];
      double pre = h2d(sp<uint16_t>(sm, s.bc_convb)[i]);
      pre = fma(h2d(cw[0]), double(c0), pre);
      pre = fma(h2d(cw[1]), double(c1), pre);
      pre = fma(h2d(cw[2]), double(c2), pre);
      pre = fma(h2d(cw[3]), y, pre);
      const double xc = silu_d(pre);
      bcx[i] = xc;
      if (w.c == 0) {
        bcst_new[i] = c1;
        bcst_new[2 * a.N + i] = c2;
        bcst_new[4 * a.N + i] = float(y);
        if (diag) {
          a.d_zx[2 * a.E + i] = y;
          a.d_xc[a.E + i] = xc;
        }
      }
    }
    csync();
    // ---- SSM update of own rows; publish g
    {
      const float* st = sp<float>(sm, s.state);
      for (int rr = warp; rr < w.nu * 16; rr += kPWarps) {
        const int u = rr / 16, r = rr % 16;
        const int e = 16 * (w.u0 + u) + r;          // row of d_inner
        const int hi = e / a.P - w.h0;
        const double dt = dt_h[hi], dA = dA_h[hi];
        const double x = yin[(xslot + u) * 16 + r];
        const double gate = yin[(zslot + u) * 16 + r];
        const double xdt = x * dt;
        const float* hrow = st + size_t(rr) * a.N;
        float* grow = L.ssm_state + size_t(e) * a.N;
        double y = 0.0;
        for (int n = lane; n < a.N; n += 32) {
          const double hv = fma(dA, double(hrow[n]), xdt * bcx[n]);
          y = fma(bcx[a.N + n], hv, y);
          grow[n] = float(hv);
        }
        y = warp_sum_d(y);
        if (lane == 0) {
          y = fma(double(sp<float>(sm, s.hd_d)[e / a.P]), x, y);
          const float gv = float(y * gate);
          tw_put(a.x_g + e, __float_as_uint(gv), tag(l, XG));
          if (diag) a.d_g[e] = gv;
        }
      }
    }
    csync();
    if (tid == 0) mbar_arrive(empty_ab);      // AB group consumed: the producer may refill it
    // ---- G: gather the gated value, gated RMSNorm
    if (!tw_gather(status, ctl, a.x_g, a.E, tag(l, XG), reinterpret_cast<uint32_t*>(gbuf), 64u)) { alive = false; break; }
    if (w.c == 0) {   // B/C conv state of this layer: every block has finished reading it
      for (int i = tid; i < 2 * a.N; i += kPThreads)
        for (int r = 0; r < 3; ++r) L.conv_state[size_t(r) * a.C + a.E + i] = bcst_new[r * 2 * a.N + i];
    }
    if (!mbar_wait_compute(status, ctl, full_cd, par, 128u)) { alive = false; break; }
    const float sx_out = prep_activation(gbuf, sp<uint16_t>(sm, s.gnorm), a.E, lora_block || wdiag, x16, xq, dg, tsum,
                                         redd, redf, redi,
                                         wdiag ? a.d_x_out : nullptr, wdiag ? a.d_xq_out : nullptr,
                                         wdiag ? a.d_xd_out : nullptr, wdiag ? a.d_xdsum_out : nullptr,
                                         wdiag ? a.d_sx_out : nullptr);
    if (a.R && warp == 0) {
      const int j = first_lora_row(a);
      if (j < a.R) {
        int acc;
        double u;
        lora_row(sp<int8_t>(sm, s.a_out), xq, a.E, sx_out, sp<uint16_t>(sm, s.sa_out)[j], &acc, &u);
        if (lane == 0) {
          tw_put_f64(a.x_uout + 2 * j, u, tag(l, XUOUT));
          if (diag) { a.d_acc_out[j] = acc; a.d_u_out[j] = u; }
        }
      }
    }
    // ---- out_proj scaffold on own tile
    int nch_out = 1;
    if (w.out_tile >= 0) nch_out = scaffold_mma(sm + s.out_tile, 1, a.kg_out, dg, a.E, part);
    if (a.R) {
      if (!tw_gather(status, ctl, a.x_uout, 2 * a.R, tag(l, XUOUT), scratch32, 256u)) { alive = false; break; }
      if (tid < a.R) u_out[tid] = f64_of(scratch32 + 2 * tid);
      csync();
      if (w.out_tile >= 0) lora2_rows(sp<int8_t>(sm, s.out_bq), 16, u_out, a.R, lo);
      csync();
    }
    // ---- residual rows, publish R of the next layer
    const bool last = (l + 1 == a.n_layer);
    if (w.out_tile >= 0) {
      if (tid < 16) {
        const int o = w.out_tile * 16 + tid;
        double y = h2d(sp<uint16_t>(sm, s.out_alpha)[tid]) * tile_row_value(part, 0, nch_out, tid, tsum);
        if (a.R) y = fma(h2d(sp<uint16_t>(sm, s.out_sb)[tid]), lo[tid], y);
        const float rn = float(double(res[o]) + y);
        if (!(last && a.layer_mode)) tw_put(a.x_r + o, __float_as_uint(rn), tag(l + 1, XR));
        if (last) {
          if (a.layer_mode) a.residual[o] = rn;
          else a.d_res[o] = rn;
        }
      }
    } else if (tid == 0 && !(last && a.layer_mode)) {
      tw_put(a.x_r + a.D + (w.c - a.out_tiles), 0u, tag(l + 1, XR));
    }
    csync();
    if (tid == 0) mbar_arrive(empty_cd);      // CD group consumed
  }

  // ---- LM head
  if (alive && !a.layer_mode) {
    const int L = a.n_layer;
    if (tw_gather(status, ctl, a.x_r, a.D + G - a.out_tiles, tag(L, XR), reinterpret_cast<uint32_t*>(res), 512u)) {
      double ss = 0.0;
      for (int k = tid; k < a.D; k += kPThreads) ss = fma(double(res[k]), double(res[k]), ss);
      ss = csum_d(ss, redd);
      const double rs = 1.0 / sqrt(ss / double(a.D) + kEpsD);
      for (int k = tid; k < a.D; k += kPThreads) gbuf[k] = float((double(res[k]) * rs) * h2d(a.normf_w[k]));
      csync();
      float best = -INFINITY;
      int besti = 0x7fffffff;
      float* hsum = sp<float>(sm, s.part);     // [kHeadChunkRows][2]
      for (int ci = 0; ci < head_chunks && alive; ++ci) {
        const int b = ci & 1;
        if (!mbar_wait_compute(status, ctl, full_h + b, unsigned(ci >> 1) & 1u, 1024u)) { alive = false; break; }
        const int r0 = v0 + ci * kHeadChunkRows, nr = min(kHeadChunkRows, v1 - r0);
        const int row = warp & (kHeadChunkRows - 1), half = warp / kHeadChunkRows;
        if (row < nr) {
          const uint4* wr = reinterpret_cast<const uint4*>(sm + size_t(b) * kHeadChunkRows * head_row_bytes +
                                                           size_t(row) * head_row_bytes);
          const int n16 = a.D / 8, hlo = half * n16 / 2, hhi = (half + 1) * n16 / 2;
          float acc = 0.f;
          for (int c = hlo + lane; c < hhi; c += 32) {
            const uint4 wv = wr[c];
            const __half2* wh = reinterpret_cast<const __half2*>(&wv);
            const float4 x0 = reinterpret_cast<const float4*>(gbuf + c * 8)[0];
            const float4 x1 = reinterpret_cast<const float4*>(gbuf + c * 8)[1];
            float2 f;
            f = __half22float2(wh[0]); acc = fmaf(f.x, x0.x, acc); acc = fmaf(f.y, x0.y, acc);
            f = __half22float2(wh[1]); acc = fmaf(f.x, x0.z, acc); acc = fmaf(f.y, x0.w, acc);
            f = __half22float2(wh[2]); acc = fmaf(f.x, x1.x, acc); acc = fmaf(f.y, x1.y, acc);
            f = __half22float2(wh[3]); acc = fmaf(f.x, x1.z, acc); acc = fmaf(f.y, x1.w, acc);
          }
          acc = warp_sum(acc);
          if (lane == 0) hsum[row * 2 + half] = acc;
        }
        csync();
        if (tid == 0) mbar_arrive(empty_h + b);
        if (tid < nr) {
          const float lg = hsum[tid * 2] + hsum[tid * 2 + 1];
          if (a.logits) a.logits[r0 + tid] = lg;
          if (lg > best || (lg == best && r0 + tid < besti)) { best = lg; besti = r0 + tid; }
        }
        csync();
      }
      // best over the threads that held rows
      if (tid < kHeadChunkRows) {
        scratch32[2 * tid] = __float_as_uint(best);
        scratch32[2 * tid + 1] = uint32_t(besti);
      }
      csync();
      if (tid == 0) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int i = 0; i < kHeadChunkRows; ++i) {
          const float v = __uint_as_float(scratch32[2 * i]);
          const int id = int(scratch32[2 * i + 1]);
          if (v > bv || (v == bv && id < bi)) { bv = v; bi = id; }
        }
        tw_put(a.x_head + 2 * w.c, __float_as_uint(bv), tag(L, XHEAD));
        tw_put(a.x_head + 2 * w.c + 1, uint32_t(bi), tag(L, XHEAD));
      }
      if (w.c == 0 && alive) {
        if (tw_gather(status, ctl, a.x_head, 2 * G, tag(L, XHEAD), scratch32, 2048u) && tid == 0) {
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
  // ---- end of token: block 0 advances the launch epoch once every block has
  // published into the last exchange (so all have read the epoch)
  if (w.c == 0 && tid == 0 && !aborted(ctl)) ctl[0] = ctl[0] + 1;
}

// ------------------------------------------------------------------ host side

inline size_t persistent_exchange_words(int D, int E, int N, int R, int grid) {
  return size_t(D + grid) + E + 4 * N + 2 * R + 2 * R + 2 * grid;
}

inline size_t persistent_scratch_bytes(int batch, int d_model, int d_inner, int in_rows, int head_blocks) {
  (void)in_rows;
  // multi-launch LM-head partials + persistent control words + exchange words (upper bounds)
  const size_t head = size_t(8) * (batch > 0 ? batch : 1) * (head_blocks > 0 ? head_blocks : 1);
  const size_t words = persistent_exchange_words(d_model, d_inner, 256, 128, 1024);
  return head + 256 + 8 * words + 256;
}

}  // namespace dfssm
