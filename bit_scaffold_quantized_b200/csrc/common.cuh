// Shared device helpers for the DF-SSM decode kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define DFSSM_DEV __device__ __forceinline__

namespace dfssm {

constexpr int kTileRows = 16;    // rows per tiled sign tile (m16n8k16 M)
constexpr int kTileCols = 256;   // columns per tiled sign tile
constexpr int kTileWords = 128;  // 32 lanes x 4 words
constexpr int kConvW = 4;        // supported conv width
constexpr float kEps = 1e-5f;    // RMSNorm epsilon
constexpr double kEpsD = 1e-5;   // RMSNorm epsilon, fp64 paths

DFSSM_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

DFSSM_DEV int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

DFSSM_DEV double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

DFSSM_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reductions with a fixed tree (deterministic); `red` holds >= 32 entries.
DFSSM_DEV double block_sum_d(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = (lane < nw) ? red[lane] : 0.0;
  t = warp_sum_d(t);
  return t;
}

DFSSM_DEV float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = (lane < nw) ? red[lane] : 0.f;
  t = warp_max(t);
  return t;
}

DFSSM_DEV float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }
DFSSM_DEV uint16_t f2h(float f) { return __half_as_ushort(__float2half_rn(f)); }

DFSSM_DEV double h2d(uint16_t h) { return double(__half2float(__ushort_as_half(h))); }

// Round-to-nearest-even fp64 -> fp16 in one step (no double rounding through fp32).
DFSSM_DEV uint16_t d2h(double v) {
  uint16_t r;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(r) : "d"(v));
  return r;
}

DFSSM_DEV double silu_d(double v) { return v / (1.0 + exp(-v)); }

DFSSM_DEV double softplus_d(double v) { return v > 20.0 ? v : log1p(exp(v)); }

// Scaffold signs as 0/1 bytes: A-fragment register of product s from tiled word q.
DFSSM_DEV uint32_t sign_bytes(uint32_t word, int s) { return (word >> s) & 0x01010101u; }

// D += A(16x32, s8, row) * B(32x8, s8, col), exact s32 accumulators.
DFSSM_DEV void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four int8 values (little-endian in a word) as two fp16 pairs, exactly: each
// byte x + 128 goes into the low mantissa byte of 1024.0 (fp16 0x6400 | u = 1024 + u)
// and 1152 = 1024 + 128 is subtracted.  lo = (x0, x1), hi = (x2, x3).
DFSSM_DEV void i8x4_to_half2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const __half2 off = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
  const uint32_t a = __byte_perm(u, 0x64646464u, 0x4140);
  const uint32_t b = __byte_perm(u, 0x64646464u, 0x4342);
  const __half2 ha = __hsub2(*reinterpret_cast<const __half2*>(&a), off);
  const __half2 hb = __hsub2(*reinterpret_cast<const __half2*>(&b), off);
  lo = *reinterpret_cast<const uint32_t*>(&ha);
  hi = *reinterpret_cast<const uint32_t*>(&hb);
}

// Eight int8 values (little-endian in a uint2) as floats, exactly, without the
// integer-to-float conversion unit (a quarter of the FMA rate): the byte c + 128
// becomes the low mantissa byte of 2^23 (float bits 0x4B0000uu = 2^23 + c + 128) and
// 2^23 + 128 is subtracted -- exact, as both operands lie within a factor of two.
DFSSM_DEV void i8x8_to_float(uint2 v, float (&f)[8]) {
  const uint32_t x = v.x ^ 0x80808080u, y = v.y ^ 0x80808080u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[i] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7440u | unsigned(i))) - 8388736.f;
    f[4 + i] = __uint_as_float(__byte_perm(y, 0x4B000000u, 0x7440u | unsigned(i))) - 8388736.f;
  }
}

// D (s32 16x8) += A (u8 16x32, row) * B (s8 32x8, col).
DFSSM_DEV void mma_u8s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D (fp32 16x8) += A (fp16 16x16, row) * B (fp16 16x8, col).
DFSSM_DEV void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Exact activation digits: an fp16 value times 2^24 is an integer X with
// |X| < 2^40; it is written as kDigits balanced base-256 digits in [-128, 127],
// X = sum_d D_d 256^d.  The scaffold sum over 0/1 sign bytes of each digit
// plane is then exact in int32, and recombining the planes in int64 gives the
// exact dot product of the +/-1 row with the fp16 activations.
constexpr int kDigits = 6;

// Exact fp16 -> fp32 by bit construction for normal values (no convert
// instruction); zero, subnormal and non-finite values take the hardware path.
DFSSM_DEV float half_to_float_bits(uint32_t h) {
  const uint32_t e = (h >> 10) & 0x1fu;
  if (e == 0u || e == 31u) return h2f(uint16_t(h));
  return __uint_as_float(((h & 0x8000u) << 16) | ((e + 112u) << 23) | ((h & 0x3ffu) << 13));
}

// x * 2^24 as an integer, exact for every finite fp16 (|X| < 2^40).
DFSSM_DEV long long half_times_2p24_64(uint32_t h) {
  const uint32_t e = (h >> 10) & 0x1fu, m = h & 0x3ffu;
  const long long X = e == 0u ? (long long)m : ((long long)(m | 0x400u) << (e - 1u));
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

// int8 activation code, decided in fp32: clamp(rint(x / sx), -127, 127) with the
// IEEE fp32 divide.  The product x * rcp (rcp = 1/sx rounded) is within
// 3 * 2^-24 |x/sx| of the correctly rounded quotient, so the divide is only needed
// near a half-integer.
DFSSM_DEV int quant_code_bits(float x, float sx, float rcp) {
  const float t = x * rcp;
  float r;
  int q = rint_small(t, &r);
  if (fabsf(fabsf(t - r) - 0.5f) <= 4.0e-5f) q = __float2int_rn(__fdiv_rn(x, sx));
  return max(-127, min(127, q));
}

// Balanced base-256 digits of X = x * 2^24 for one fp16 value, packed: planes 0-3
// in `lo` (byte d = digit d), planes 4-5 in the low two bytes of `hi`.
DFSSM_DEV void digits_of(uint32_t h, uint32_t* lo, uint32_t* hi) {
  if ((h & 0x7fffu) <= 0x57f0u) {          // |x| <= 127: |X| < 2^31, four digits
    const uint32_t e = (h >> 10) & 0x1fu, m = h & 0x3ffu;
    int X = e == 0u ? int(m) : int((m | 0x400u) << (e - 1u));
    X = (h & 0x8000u) ? -X : X;
    *lo = (uint32_t(X) + 0x80808080u) ^ 0x80808080u;
    *hi = 0u;
    return;
  }
  long long X = half_times_2p24_64(h);
  uint32_t b[kDigits];
#pragma unroll
  for (int d = 0; d < kDigits; ++d) {
    const long long Dd = ((X + 128) & 255) - 128;
    b[d] = uint32_t(Dd) & 0xffu;
    X = (X - Dd) >> 8;
  }
  *lo = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
  *hi = b[4] | (b[5] << 8);
}

// ---- mbarriers and bulk copies (global -> this CTA's shared memory)

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
// Transaction bytes without an arrival (a second part of a phase's copies announced
// after the arrival that armed it, or before it).
DFSSM_DEV void mbar_expect_tx_only(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the kernel before it on the stream still runs: it
// may read only data that no earlier kernel of the sequence writes (weights) before
// pdl_wait(), which returns once every earlier kernel has completed and its writes
// are visible (at once for an ordinary launch); pdl_release() lets the next kernel
// start its own setup.
DFSSM_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
DFSSM_DEV void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Generic-proxy writes of this thread to shared memory become visible to later
// bulk copies (async proxy) that read them.
DFSSM_DEV void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

DFSSM_DEV uint32_t cluster_map(uint32_t saddr, unsigned rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Every thread of every CTA of the cluster.
DFSSM_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

DFSSM_DEV void st_cluster_f64(uint32_t addr, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" :: "r"(addr), "d"(v) : "memory");
}
DFSSM_DEV void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(addr), "r"(v) : "memory");
}

}  // namespace dfssm
