// DF-SSM decode-step kernels ("Density Field State Space Models", Section 3.2 Eq. 3,
// Section 3.3, Section 4.1, Appendix B), multi-launch path (any batch), one launch
// per stage:
//   k_prologue_cl   RMSNorm -> fp16 activation -> int8 codes, digit planes -> LoRA
//                   stage 1 (A_q . x_q); one cluster of 4 CTAs per batch row
//   k_proj          1-bit scaffold on int8 tensor cores (0/1 sign bytes x exact
//                   activation digit planes, exact integer accumulation) + LoRA stage 2
//                   (fp64) + epilogue (store | residual add | conv1d step + step sizes)
//   k_ssm_stream    selective-SSM state update + D skip + gate y * silu(z), state items
//                   streamed through shared memory by bulk copies (k_ssm: large items)
//   k_lmhead_tc     final RMSNorm + tied LM head (fp16 or int8 rows) on tensor cores +
//                   per-block argmax (k_lmhead: fp32 fallback); k_argmax finishes it
//   k_embed, k_quant_rows, k_pack_*   embedding gather, int8 row quantiser, sign packing
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace dfssm {

// ------------------------------------------------------------------ packing

DFSSM_DEV float load_dense(const void* w, int dtype, size_t i) {
  return dtype == 0 ? h2f(reinterpret_cast<const uint16_t*>(w)[i])
                    : reinterpret_cast<const float*>(w)[i];
}

// Inverse of the tiled layout: (tile word, bit) -> (row, col) inside the matrix.
// Word q of a lane holds register q of the A fragments of the tile's eight
// 32-column m16n8k32 .s8 products s = 0..7: bit s + 8 i is byte i of that register
// (m16n8k32 .s8 fragment: rows g / g+8, columns 4t + i / 16 + 4t + i of the
// product).  Product s = 2 m + e covers tile columns 64 m + 16 t + 8 e + [0, 8) of
// lane t, so the B bytes of products 2m and 2m + 1 are 16 consecutive columns.
DFSSM_DEV void tiled_coord(size_t word, int bit, int kgroups, int* row, int* col) {
  const size_t tile = word / kTileWords;
  const int within = int(word % kTileWords);
  const int lane = within >> 2, q = within & 3;
  const int rt = int(tile / kgroups), kg = int(tile % kgroups);
  const int s = bit & 7, i = bit >> 3;
  const int g = lane >> 2, t = lane & 3;
  *row = rt * kTileRows + g + 8 * (q & 1);
  *col = kg * kTileCols + 64 * (s >> 1) + 16 * t + 8 * (s & 1) + 4 * (q >> 1) + i;
}

__global__ void k_pack_rowmajor(const void* __restrict__ w, int dtype, int rows, int cols,
                                uint32_t* __restrict__ bits) {
  const int wpr = cols / 32;
  const size_t n = size_t(rows) * wpr;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += size_t(gridDim.x) * blockDim.x) {
    const size_t r = i / wpr, kw = i % wpr;
    uint32_t word = 0;
    for (int j = 0; j < 32; ++j)
      word |= (load_dense(w, dtype, r * cols + kw * 32 + j) >= 0.f ? 1u : 0u) << j;
    bits[i] = word;
  }
}

__global__ void k_pack_tiled(const void* __restrict__ w, int dtype, int rows, int cols,
                             uint32_t* __restrict__ bits, size_t nwords) {
  const int kgroups = cols / kTileCols;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords;
       i += size_t(gridDim.x) * blockDim.x) {
    uint32_t word = 0;
    for (int b = 0; b < 32; ++b) {
      int r, c;
      tiled_coord(i, b, kgroups, &r, &c);
      if (r < rows && load_dense(w, dtype, size_t(r) * cols + c) >= 0.f) word |= 1u << b;
    }
    bits[i] = word;
  }
}

__global__ void k_repack_tiled(const uint32_t* __restrict__ src, int rows, int cols,
                               uint32_t* __restrict__ bits, size_t nwords) {
  const int kgroups = cols / kTileCols, wpr = cols / 32;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords;
       i += size_t(gridDim.x) * blockDim.x) {
    uint32_t word = 0;
    for (int b = 0; b < 32; ++b) {
      int r, c;
      tiled_coord(i, b, kgroups, &r, &c);
      if (r < rows && ((src[size_t(r) * wpr + c / 32] >> (c & 31)) & 1u)) word |= 1u << b;
    }
    bits[i] = word;
  }
}

// ------------------------------------------------------------------ prologue

struct PrologueArgs {
  int K, rank;
  const float* src;       // mode 0: [B][K] fp32 value to normalise (residual or gated value)
  const uint16_t* src16;  // mode 1: fp16 [B][K] activation as given
  const uint16_t* w;      // fp16 [K] norm weight (mode 0)
  uint16_t* x;            // fp16 [B][K] out (mode 0; may be null)
  int8_t* xq;             // int8 [B][K] LoRA codes out
  float* sx;              // fp32 [B] out
  int8_t* xd;             // int8 [B][kDigits][K] scaffold digit planes out
  int* xdsum;             // int32 [B][kDigits] digit-plane sums out
  const int8_t* A;        // int8 [rank][K]
  const uint16_t* sA;     // fp16 [rank]
  int* acc;               // int32 [B][rank] out
  double* u;              // fp64 [B][rank] out
};

// Cluster prologue: one cluster of kPrologueCQ CTAs per batch row (grid (CQ, B));
// CTA rank q owns columns [q K/CQ, (q+1) K/CQ), at most 4 per thread.  The row's
// sum of squares and max |x| are all-reduced through distributed shared memory
// (each CTA stores its partial into every CTA; all sum in rank order, so every CTA
// holds the same value); each CTA writes its columns' x, codes and digit planes;
// the digit-plane sums and the LoRA stage-1 partials of its columns go to rank 0,
// which adds them in rank order (exact) and writes xdsum, acc, u and sx.
// Arithmetic:
//   mode 0: x = fp16(src * (1/sqrt(mean(src^2) + eps)) * w), all in fp64
//   mode 1: x = src16
//   sx = max|x| / 127, xq = clamp(rint(x / sx), -127, 127) (fp32 decision)
//   acc[j] = sum_k A[j,k] xq[k] (exact), u[j] = acc[j] * sA[j] * sx (fp64)
constexpr int kPrologueCQ = 4;
constexpr int kPrologueClThreads = 512;  // two CTAs per SM (64 registers): a batch of 64 rows runs in one wave
constexpr int kPrologueClVals = 4;      // K / CQ / 512 <= 4: K <= 8192
constexpr int kPrologueMaxRank = 128;

// V = ceil(K / CQ / 512) values per thread (no padding values through the
// normalisation's slow path).
template <int MODE, int V>
__global__ void __cluster_dims__(kPrologueCQ, 1, 1) __launch_bounds__(kPrologueClThreads, 2)
    k_prologue_cl(PrologueArgs a) {
  constexpr int CQ = kPrologueCQ, NW = kPrologueClThreads / 32;
  __shared__ double xss[CQ];
  __shared__ float xam[CQ];
  __shared__ int xpart[CQ][kDigits + kPrologueMaxRank];
  __shared__ double redd[32];
  __shared__ float red[32];
  __shared__ int red6[NW][kDigits];
  __shared__ __align__(16) int8_t qs[8192 / CQ];
  const int K = a.K, Kq = K / CQ;
  const int q = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = q * Kq;

  // this warp's first two LoRA rows over the CTA's columns (loads issued first)
  const int nvq = Kq / 16;                                  // 16-byte chunks of a row slice (<= 128)
  uint4 av[2][4];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int j = warp + NW * rr, c = lane + 32 * m;
      av[rr][m] = (j < a.rank && c < nvq) ? __ldg(reinterpret_cast<const uint4*>(a.A + size_t(j) * K + k0) + c)
                                          : make_uint4(0, 0, 0, 0);
    }
  pdl_wait();                              // the source row is the previous kernel's output
  pdl_release();
  uint32_t h[V];
  float am = 0.f;
  if (MODE == 0) {
    const float* v = a.src + size_t(b) * K + k0;
    float vf[V];
    uint16_t wh[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int k = tid + i * kPrologueClThreads;
      vf[i] = k < Kq ? v[k] : 0.f;
      wh[i] = k < Kq ? a.w[k0 + k] : uint16_t(0);
    }
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < V; ++i) ss = fma(double(vf[i]), double(vf[i]), ss);
    ss = block_sum_d(ss, redd);
    cluster_sync_all();                    // every CTA of the cluster runs: remote stores allowed
    if (tid < CQ) st_cluster_f64(cluster_map(smem_u32(&xss[q]), tid), ss);
    cluster_sync_all();
    double sst = 0.0;
#pragma unroll
    for (int r = 0; r < CQ; ++r) sst += xss[r];
    const double rs = 1.0 / sqrt(sst / double(K) + kEpsD);
    const float rs32 = float(rs);
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int k = tid + i * kPrologueClThreads;
      h[i] = 0u;
      if (k >= Kq) continue;
      h[i] = norm_fp16(vf[i], rs, rs32, half_to_float_bits(wh[i]));
      am = fmaxf(am, fabsf(half_to_float_bits(h[i])));
      if (a.x) a.x[size_t(b) * K + k0 + k] = uint16_t(h[i]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int k = tid + i * kPrologueClThreads;
      h[i] = k < Kq ? a.src16[size_t(b) * K + k0 + k] : 0u;
      am = fmaxf(am, fabsf(half_to_float_bits(h[i])));
    }
    cluster_sync_all();                    // every CTA of the cluster runs: remote stores allowed
  }
  am = block_max(am, red);
  if (tid < CQ) st_cluster_u32(cluster_map(smem_u32(&xam[q]), tid), __float_as_uint(am));
  cluster_sync_all();
  float amt = 0.f;
#pragma unroll
  for (int r = 0; r < CQ; ++r) amt = fmaxf(amt, xam[r]);
  const float sx = amt > 0.f ? __fdiv_rn(amt, 127.f) : 1.f;
  const float rcp = __frcp_rn(sx);
  int dsum[kDigits];
#pragma unroll
  for (int d = 0; d < kDigits; ++d) dsum[d] = 0;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int k = tid + i * kPrologueClThreads;
    if (k < Kq) {
      const int8_t c = amt > 0.f ? int8_t(quant_code_bits(half_to_float_bits(h[i]), sx, rcp)) : int8_t(0);
      qs[k] = c;
      a.xq[size_t(b) * K + k0 + k] = c;
      uint32_t lo, hi;
      digits_of(h[i], &lo, &hi);
      const uint32_t w6[kDigits] = {lo, lo >> 8, lo >> 16, lo >> 24, hi, hi >> 8};
#pragma unroll
      for (int d = 0; d < kDigits; ++d) {
        const int8_t dg = int8_t(w6[d] & 0xffu);
        a.xd[(size_t(b) * kDigits + d) * K + k0 + k] = dg;
        dsum[d] += dg;
      }
    }
  }
#pragma unroll
  for (int d = 0; d < kDigits; ++d) {
    const int t = __reduce_add_sync(0xffffffffu, dsum[d]);
    if (lane == 0) red6[warp][d] = t;
  }
  __syncthreads();                         // codes and the warps' plane sums complete
  if (tid < kDigits) {
    int t = 0;
    for (int w = 0; w < NW; ++w) t += red6[w][tid];
    st_cluster_u32(cluster_map(smem_u32(&xpart[q][tid]), 0), uint32_t(t));
  }
  // LoRA stage-1 partials of this CTA's columns: warp w takes rows w, w + 16, ...
  const uint4* q16 = reinterpret_cast<const uint4*>(qs);
  for (int j = warp, rr = 0; j < a.rank; j += NW, ++rr) {
    int acc = 0;
    if (rr < 2) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int c = lane + 32 * m;
        if (c < nvq) {
          const uint4 x4 = q16[c], w4 = rr == 0 ? av[0][m] : av[1][m];
          acc = __dp4a(int(w4.x), int(x4.x), acc);
          acc = __dp4a(int(w4.y), int(x4.y), acc);
          acc = __dp4a(int(w4.z), int(x4.z), acc);
          acc = __dp4a(int(w4.w), int(x4.w), acc);
        }
      }
    } else {
      for (int c = lane; c < nvq; c += 32) {
        const uint4 x4 = q16[c], w4 = __ldg(reinterpret_cast<const uint4*>(a.A + size_t(j) * K + k0) + c);
        acc = __dp4a(int(w4.x), int(x4.x), acc);
        acc = __dp4a(int(w4.y), int(x4.y), acc);
        acc = __dp4a(int(w4.z), int(x4.z), acc);
        acc = __dp4a(int(w4.w), int(x4.w), acc);
      }
    }
    acc = warp_sum_i(acc);
    if (lane == 0) st_cluster_u32(cluster_map(smem_u32(&xpart[q][kDigits + j]), 0), uint32_t(acc));
  }
  cluster_sync_all();                      // rank 0 holds every CTA's partials
  if (q == 0) {
    if (tid < kDigits) {
      int t = 0;
      for (int r = 0; r < CQ; ++r) t += xpart[r][tid];
      a.xdsum[b * kDigits + tid] = t;
      if (tid == 0) a.sx[b] = sx;
    }
    for (int j = tid; j < a.rank; j += kPrologueClThreads) {
      int acc = 0;
      for (int r = 0; r < CQ; ++r) acc += xpart[r][kDigits + j];
      a.acc[size_t(b) * a.rank + j] = acc;
      a.u[size_t(b) * a.rank + j] = (double(acc) * h2d(a.sA[j])) * double(sx);
    }
  }
}

// Row prologue: the same outputs as k_prologue_cl from one 512-thread CTA per batch
// row (grid (B)), for batches that fill the GPU with rows: no cluster exchange, three
// block barriers.  Thread t owns the 4-column groups t, t + 512, ... (16-byte loads,
// one word per group and output plane); warp w takes LoRA rows w, w + 16, ... (the
// first two rows' slices loaded up front, later rows' chunks all requested before
// their products).  The sum of squares and max |x| are reduced by
// every warp from the 16 warp partials in a fixed order.
constexpr int kPrologueRowThreads = 512;
constexpr int kPrologueRowGroups = 4;    // 4-column groups per thread: K <= 8192
constexpr int kPrologueRowMinBatch = 16;

// G = ceil(K / 2048) groups per thread, so that no thread carries padding columns
// through the normalisation (a zero takes the slow exact-rounding path).
template <int MODE, int G>
__global__ void __launch_bounds__(kPrologueRowThreads, 1) k_prologue_row(PrologueArgs a) {
  constexpr int NW = kPrologueRowThreads / 32, PRE = G < 2 ? 4 : 8;   // chunks per lane of a row: K / 512
  __shared__ double redd[NW];
  __shared__ float redf[NW];
  __shared__ int red6[NW][kDigits];
  __shared__ __align__(16) int8_t qs[8192];
  const int K = a.K, b = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nvq = K / 16;                                   // 16-byte chunks of a row
  // the warp's first two LoRA rows (all of them up to rank 32), up to K = 4096, are
  // requested before any arithmetic
  uint4 av[2][PRE];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr)
#pragma unroll
    for (int m = 0; m < PRE; ++m) {
      const int c = lane + 32 * m, j = warp + NW * rr;
      av[rr][m] = (j < a.rank && c < nvq) ? __ldg(reinterpret_cast<const uint4*>(a.A + size_t(j) * K) + c)
                                          : make_uint4(0, 0, 0, 0);
    }
  pdl_wait();                              // the source row is the previous kernel's output
  pdl_release();
  uint32_t h[G][4];
  float am = 0.f;
  if (MODE == 0) {
    float vf[G][4];
    uint2 wh[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int k = 4 * (tid + kPrologueRowThreads * g);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      uint2 w = make_uint2(0u, 0u);
      if (k < K) {
        v = *reinterpret_cast<const float4*>(a.src + size_t(b) * K + k);
        w = *reinterpret_cast<const uint2*>(a.w + k);
      }
      vf[g][0] = v.x; vf[g][1] = v.y; vf[g][2] = v.z; vf[g][3] = v.w;
      wh[g] = w;
    }
    double ss = 0.0;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) ss = fma(double(vf[g][e]), double(vf[g][e]), ss);
    ss = warp_sum_d(ss);
    if (lane == 0) redd[warp] = ss;
    __syncthreads();
    const double sst = warp_sum_d(lane < NW ? redd[lane] : 0.0);
    const double rs = 1.0 / sqrt(sst / double(K) + kEpsD);
    const float rs32 = float(rs);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int k = 4 * (tid + kPrologueRowThreads * g);
      const uint32_t wv[4] = {wh[g].x & 0xffffu, wh[g].x >> 16, wh[g].y & 0xffffu, wh[g].y >> 16};
#pragma unroll
      for (int e = 0; e < 4; ++e) h[g][e] = 0u;
      if (k >= K) continue;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        h[g][e] = norm_fp16(vf[g][e], rs, rs32, half_to_float_bits(wv[e]));
        am = fmaxf(am, fabsf(half_to_float_bits(h[g][e])));
      }
      if (a.x)
        *reinterpret_cast<uint2*>(a.x + size_t(b) * K + k) =
            make_uint2(h[g][0] | (h[g][1] << 16), h[g][2] | (h[g][3] << 16));
    }
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int k = 4 * (tid + kPrologueRowThreads * g);
      uint2 v = make_uint2(0u, 0u);
      if (k < K) v = *reinterpret_cast<const uint2*>(a.src16 + size_t(b) * K + k);
      h[g][0] = v.x & 0xffffu; h[g][1] = v.x >> 16; h[g][2] = v.y & 0xffffu; h[g][3] = v.y >> 16;
#pragma unroll
      for (int e = 0; e < 4; ++e) am = fmaxf(am, fabsf(half_to_float_bits(h[g][e])));
    }
  }
  am = warp_max(am);
  if (lane == 0) redf[warp] = am;
  __syncthreads();
  const float amt = warp_max(lane < NW ? redf[lane] : 0.f);
  const float sx = amt > 0.f ? __fdiv_rn(amt, 127.f) : 1.f;
  const float rcp = __frcp_rn(sx);
  int dsum[kDigits];
#pragma unroll
  for (int d = 0; d < kDigits; ++d) dsum[d] = 0;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int k = 4 * (tid + kPrologueRowThreads * g);
    if (k < K) {
      uint32_t cw = 0u, pw[kDigits] = {0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t c = amt > 0.f ? uint32_t(quant_code_bits(half_to_float_bits(h[g][e]), sx, rcp)) & 0xffu : 0u;
        cw |= c << (8 * e);
        uint32_t lo, hi;
        digits_of(h[g][e], &lo, &hi);
        const uint32_t w6[kDigits] = {lo, lo >> 8, lo >> 16, lo >> 24, hi, hi >> 8};
#pragma unroll
        for (int d = 0; d < kDigits; ++d) {
          pw[d] |= (w6[d] & 0xffu) << (8 * e);
          dsum[d] += int8_t(w6[d] & 0xffu);
        }
      }
      *reinterpret_cast<uint32_t*>(qs + k) = cw;
      *reinterpret_cast<uint32_t*>(a.xq + size_t(b) * K + k) = cw;
#pragma unroll
      for (int d = 0; d < kDigits; ++d)
        *reinterpret_cast<uint32_t*>(a.xd + (size_t(b) * kDigits + d) * K + k) = pw[d];
    }
  }
#pragma unroll
  for (int d = 0; d < kDigits; ++d) {
    const int t = __reduce_add_sync(0xffffffffu, dsum[d]);
    if (lane == 0) red6[warp][d] = t;
  }
  __syncthreads();                         // codes and the warps' plane sums complete
  if (tid < kDigits) {
    int t = 0;
    for (int w = 0; w < NW; ++w) t += red6[w][tid];
    a.xdsum[b * kDigits + tid] = t;
    if (tid == 0) a.sx[b] = sx;
  }
  const uint4* q16 = reinterpret_cast<const uint4*>(qs);
  auto dot4 = [](const uint4& w4, const uint4& x4, int acc) {
    acc = __dp4a(int(w4.x), int(x4.x), acc);
    acc = __dp4a(int(w4.y), int(x4.y), acc);
    acc = __dp4a(int(w4.z), int(x4.z), acc);
    return __dp4a(int(w4.w), int(x4.w), acc);
  };
  for (int rr = 0, j = warp; j < a.rank; ++rr, j += NW) {
    int acc = 0;
    if (rr < 2) {
#pragma unroll
      for (int m = 0; m < PRE; ++m) {
        const int c = lane + 32 * m;
        if (c < nvq) acc = dot4(rr == 0 ? av[0][m] : av[1][m], q16[c], acc);
      }
      for (int c = lane + 32 * PRE; c < nvq; c += 32)
        acc = dot4(__ldg(reinterpret_cast<const uint4*>(a.A + size_t(j) * K) + c), q16[c], acc);
    } else {
      // later rows (rank > 32): every chunk of the row requested before the products
      uint4 w[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int c = lane + 32 * m;
        w[m] = c < nvq ? __ldg(reinterpret_cast<const uint4*>(a.A + size_t(j) * K) + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int c = lane + 32 * m;
        if (c < nvq) acc = dot4(w[m], q16[c], acc);
      }
    }
    acc = warp_sum_i(acc);
    if (lane == 0) {
      a.acc[size_t(b) * a.rank + j] = acc;
      a.u[size_t(b) * a.rank + j] = (double(acc) * h2d(a.sA[j])) * double(sx);
    }
  }
}

// ------------------------------------------------------------------ projection

enum { EPI_STORE = 0, EPI_RESID = 1, EPI_INPROJ = 2, EPI_ZX = 3 };

struct ProjArgs {
  int rows, K, rank, batch;
  const uint32_t* bits;   // tiled sign words
  const uint16_t* alpha;
  const int8_t* B;        // [rows][rank]
  const uint16_t* sB;
  const int8_t* xd;       // int8 [batch][kDigits][K] activation digit planes
  const int* xdsum;       // int32 [batch][kDigits]
  const double* u;        // fp64 [batch][rank]
  float* out;             // EPI_STORE: fp32 [batch][rows]; EPI_RESID: fp32 residual [batch][rows]
  double* zx;             // EPI_INPROJ, EPI_ZX: fp64 [batch][rows]
  // EPI_INPROJ conv step over rows [conv_lo, conv_lo + conv_dim)
  int conv_lo, conv_dim;
  const uint16_t* conv_w;  // [conv_dim][4]
  const uint16_t* conv_b;  // [conv_dim]
  float* conv_state;       // fp32 [batch][3][conv_dim]
  double* xc;              // fp64 [batch][conv_dim]
  unsigned* status;        // workspace status word (value 65536: a tensor-core wait gave up), may be null
};

constexpr int kProjWarps = 16;
constexpr int kProjThreads = kProjWarps * 32;

__host__ __device__ constexpr int proj_cols(int bt) { return ((kDigits * bt + 7) / 8) * 8; }
__host__ __device__ __forceinline__ int proj_dstride(int K) { return K + 64; }  // bytes; == 64 mod 128: conflict-free 16-byte B loads
__host__ __device__ constexpr int proj_pstride(int bt) { return proj_cols(bt) + 1; }  // odd: spreads banks
__host__ __device__ __forceinline__ size_t proj_smem_bytes(int K, int rank, int bt) {
  return size_t(proj_cols(bt)) * proj_dstride(K)                 // digit planes
         + size_t(8) * bt * (rank > 0 ? rank : 1)                 // u (fp64)
         + size_t(4) * kProjWarps * 16 * proj_pstride(bt)         // per-warp int32 tile sums
         + size_t(4) * bt * kDigits;                              // digit sums
}

// Output (batch row b, projection row o) with value y: store, residual add, or the
// in_proj epilogue (fp64 store, conv step + SiLU of the conv rows, step size and
// decay of the dt rows).
template <int EPI>
DFSSM_DEV void proj_epilogue(const ProjArgs& a, int b, int o, double y) {
  const size_t oi = size_t(b) * a.rows + o;
  if (EPI == EPI_RESID) {
    a.out[oi] = float(double(a.out[oi]) + y);
  } else if (EPI == EPI_STORE) {
    a.out[oi] = float(y);
  } else if (EPI == EPI_ZX) {
    a.zx[oi] = y;
  } else {
    a.zx[oi] = y;
    const int c = o - a.conv_lo;
    if (c >= 0 && c < a.conv_dim) {
      float* cs = a.conv_state + size_t(b) * 3 * a.conv_dim;
      const uint2 wv = *reinterpret_cast<const uint2*>(a.conv_w + size_t(c) * 4);
      const double s0 = cs[c], s1 = cs[a.conv_dim + c], s2 = cs[2 * a.conv_dim + c];
      double pre = h2d(a.conv_b[c]);
      pre = fma(h2d(uint16_t(wv.x & 0xffff)), s0, pre);
      pre = fma(h2d(uint16_t(wv.x >> 16)), s1, pre);
      pre = fma(h2d(uint16_t(wv.y & 0xffff)), s2, pre);
      pre = fma(h2d(uint16_t(wv.y >> 16)), y, pre);
      a.xc[size_t(b) * a.conv_dim + c] = silu_d(pre);
      cs[c] = float(s1);
      cs[a.conv_dim + c] = float(s2);
      cs[2 * a.conv_dim + c] = float(y);
    }
  }
}

// proj_epilogue for up to M batch rows bs[0..n) of one projection row o, with every
// load the stores could alias (the residual, the conv state) issued before the first
// store, so that a thread waits for one round trip per group rather than per output.
template <int EPI, int M>
DFSSM_DEV void proj_epilogue_group(const ProjArgs& a, int o, const int (&bs)[M], const double (&ys)[M], int n) {
  if (EPI == EPI_RESID) {
    float r[M];
#pragma unroll
    for (int i = 0; i < M; ++i) r[i] = i < n ? a.out[size_t(bs[i]) * a.rows + o] : 0.f;
#pragma unroll
    for (int i = 0; i < M; ++i)
      if (i < n) a.out[size_t(bs[i]) * a.rows + o] = float(double(r[i]) + ys[i]);
  } else if (EPI == EPI_INPROJ && o - a.conv_lo >= 0 && o - a.conv_lo < a.conv_dim) {
    const int c = o - a.conv_lo, cd = a.conv_dim;
    float s0[M], s1[M], s2[M];
#pragma unroll
    for (int i = 0; i < M; ++i) {
      const float* cs = a.conv_state + size_t(i < n ? bs[i] : 0) * 3 * cd;
      s0[i] = i < n ? cs[c] : 0.f;
      s1[i] = i < n ? cs[cd + c] : 0.f;
      s2[i] = i < n ? cs[2 * cd + c] : 0.f;
    }
    const uint2 wv = *reinterpret_cast<const uint2*>(a.conv_w + size_t(c) * 4);
    const double w0 = h2d(uint16_t(wv.x & 0xffff)), w1 = h2d(uint16_t(wv.x >> 16));
    const double w2 = h2d(uint16_t(wv.y & 0xffff)), w3 = h2d(uint16_t(wv.y >> 16)), cb = h2d(a.conv_b[c]);
#pragma unroll
    for (int i = 0; i < M; ++i) {
      if (i < n) {
        const int b = bs[i];
        const double y = ys[i];
        a.zx[size_t(b) * a.rows + o] = y;
        double pre = cb;
        pre = fma(w0, double(s0[i]), pre);
        pre = fma(w1, double(s1[i]), pre);
        pre = fma(w2, double(s2[i]), pre);
        pre = fma(w3, y, pre);
        a.xc[size_t(b) * cd + c] = silu_d(pre);
        float* cs = a.conv_state + size_t(b) * 3 * cd;
        cs[c] = s1[i];
        cs[cd + c] = s2[i];
        cs[2 * cd + c] = float(y);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < M; ++i)
      if (i < n) proj_epilogue<EPI>(a, bs[i], o, ys[i]);
  }
}

// Scaffold value of one row from its per-plane 0/1 sums q[d] = sum_k bit * D_d[k]:
// sum_k s[k] x[k] = 2^-24 * sum_d 256^d (2 q[d] - T[d]), exact in int64.
DFSSM_DEV double scaffold_value(const int (&q)[kDigits], const int* T) {
  long long S = 0;
#pragma unroll
  for (int d = kDigits - 1; d >= 0; --d) S = S * 256 + (2LL * q[d] - T[d]);
  return double(S) * (1.0 / 16777216.0);
}

// grid (gx, ceil(batch/BT)), gx sized to the resident blocks.  A block stages the
// digit planes of its BT batch rows once; each warp then owns whole 16-row tiles
// (rt = 16 blockIdx.x + warp, then + 16 gridDim.x, ...) over the full K, so the
// integer sums never leave the warp and no block barrier follows the staging.  Per
// 256-column group the warp expands its lane's 16-byte vector of sign words (loaded
// two groups ahead) into 0/1 int8 A fragments (one shift + one mask per register)
// and runs m16n8k32 int8 MMAs against the planes, one 16-byte B load per plane row
// serving two products; the epilogue recombines the planes exactly (lane = row,
// batch rows split over the two half-warps) and adds the LoRA stage 2 in fp64.
template <int EPI, int BT>
__global__ void __launch_bounds__(kProjThreads) k_proj(ProjArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int NC = proj_cols(BT), NT = NC / 8, PS = proj_pstride(BT);
  const int K = a.K, DS = proj_dstride(K), rk = a.rank > 0 ? a.rank : 1;
  int8_t* dg = reinterpret_cast<int8_t*>(smem);                                   // [NC][DS]
  double* us = reinterpret_cast<double*>(smem + size_t(NC) * DS);                 // [BT][rank]
  int* part = reinterpret_cast<int*>(us + BT * rk);                               // [warps][16][PS]
  int* T = part + kProjWarps * 16 * PS;                                           // [BT][kDigits]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b0 = blockIdx.y * BT;
  pdl_wait();                              // digit planes and u come from the prologue
  pdl_release();
  const int kgroups = K / kTileCols;
  const int ntiles = (a.rows + kTileRows - 1) / kTileRows;

  // stage digit planes: column c = bb * kDigits + d (zero past the batch and past 6*BT)
  for (int i = tid; i < NC * (K / 16); i += blockDim.x) {
    const int c = i / (K / 16), c16 = i % (K / 16);
    const int bb = c / kDigits, d = c % kDigits;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (bb < BT && b0 + bb < a.batch)
      v = reinterpret_cast<const uint4*>(a.xd + (size_t(b0 + bb) * kDigits + d) * K)[c16];
    *reinterpret_cast<uint4*>(dg + size_t(c) * DS + c16 * 16) = v;
  }
  for (int i = tid; i < BT * a.rank; i += blockDim.x) {
    const int bb = i / a.rank, j = i % a.rank;
    us[i] = (b0 + bb < a.batch) ? a.u[size_t(b0 + bb) * a.rank + j] : 0.0;
  }
  for (int i = tid; i < BT * kDigits; i += blockDim.x)
    T[i] = (b0 + i / kDigits < a.batch) ? a.xdsum[size_t(b0) * kDigits + i] : 0;
  __syncthreads();

  const int g = lane >> 2, t = lane & 3;
  int* wp = part + warp * 16 * PS;
  const uint4 zero4 = make_uint4(0, 0, 0, 0);
  for (int rt = blockIdx.x * kProjWarps + warp; rt < ntiles; rt += gridDim.x * kProjWarps) {
    int acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0;
    const uint4* tiles = reinterpret_cast<const uint4*>(a.bits) + size_t(rt) * kgroups * 32 + lane;
    uint4 w0 = __ldg(tiles), w1 = kgroups > 1 ? __ldg(tiles + 32) : zero4;
    for (int kg = 0; kg < kgroups; ++kg) {
      const uint4 wv = w0;
      w0 = w1;
      w1 = kg + 2 < kgroups ? __ldg(tiles + (kg + 2) * 32) : zero4;
      const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint32_t a0[4], a1[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          a0[q] = sign_bytes(words[q], 2 * m);
          a1[q] = sign_bytes(words[q], 2 * m + 1);
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint4 bq = *reinterpret_cast<const uint4*>(dg + size_t(n * 8 + g) * DS + kg * kTileCols + 64 * m + 16 * t);
          mma_s8_16832(acc[n], a0, bq.x, bq.y);
          mma_s8_16832(acc[n], a1, bq.z, bq.w);
        }
      }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      wp[g * PS + n * 8 + 2 * t] = acc[n][0];
      wp[g * PS + n * 8 + 2 * t + 1] = acc[n][1];
      wp[(g + 8) * PS + n * 8 + 2 * t] = acc[n][2];
      wp[(g + 8) * PS + n * 8 + 2 * t + 1] = acc[n][3];
    }
    __syncwarp();

    const int r = lane & 15, o = rt * kTileRows + r;
    if (o < a.rows) {
      const int* Br4 = reinterpret_cast<const int*>(a.B + size_t(o) * a.rank);
      const double al = h2d(a.alpha[o]);
      const double sb = a.rank > 0 ? h2d(a.sB[o]) : 0.0;
      for (int bb = lane >> 4; bb < BT; bb += 2) {
        const int b = b0 + bb;
        if (b >= a.batch) break;
        int q[kDigits];
#pragma unroll
        for (int d = 0; d < kDigits; ++d) q[d] = wp[r * PS + bb * kDigits + d];
        double y = al * scaffold_value(q, T + bb * kDigits);
        if (a.rank > 0) {
          const double* ur = us + bb * a.rank;
          double l = 0.0;
          for (int j4 = 0; j4 < a.rank / 4; ++j4) {
            const int v = __ldg(Br4 + j4);
#pragma unroll
            for (int e = 0; e < 4; ++e) l = fma(double(int8_t(v >> (8 * e))), ur[4 * j4 + e], l);
          }
          y = fma(sb, l, y);
        }
        proj_epilogue<EPI>(a, b, o, y);
      }
    }
    __syncwarp();   // the warp's tile sums are consumed before its next tile's
  }
}

// ------------------------------------------------------------------ projection on tcgen05
//
// The batched scaffold on the 5th-generation tensor cores: tcgen05.mma kind::i8
// (0/1 sign bytes times signed digit-plane bytes, int32 accumulators in tensor
// memory).  A CTA owns one M = 128 tile of projection rows, a group of BG batch rows
// (N = 6 BG digit-plane columns) and a share of K: gridDim.z CTAs of one cluster
// split K and add their integer sums over distributed shared memory.  The warps
// specialise:
//   warp 0       TMA producer: per 256-column k-block, the 8 row tiles' packed sign
//                words (one 2D box of 8 x 512 bytes) and the batch rows' digit planes
//                (two 2D boxes of 128 K-bytes x N rows, 128-byte swizzle) into a ring
//                of shared-memory stages;
//   warp 1       MMA issuer (one thread): eight K = 32 MMAs per k-block, A read from
//                tensor memory and B from the stage, committed to the stage's and the
//                A buffer's `empty` barriers, the last also to `done`;
//   warps 2..5   expanders: thread = one tile row (TMEM lane); it gathers the row's
//                256 sign bits of the k-block from the stage and writes them as 0/1
//                bytes into one of four A buffers in tensor memory (64 columns each,
//                4 K-bytes per column);
//   warps 6..11  LoRA stage 2 while the MMAs run: l[row][b] = sum_j B_q[row][j] u[b][j]
//                for the rows this CTA finishes, as fp64 tensor-core MMAs (m16n8k4),
//                into shared memory;
//   warps 0..7   the epilogue: tcgen05.ld of the accumulators (warp w: TMEM lanes
//                32 (w mod 4) .. + 31 = tile rows) and each (row, batch row) finished
//                exactly as k_proj does; with a K split, each CTA folds its plane
//                sums into one int64 partial per (row, batch row) and stores it
//                (st.async) into CTA z of the cluster, which adds them for rows
//                [128 z / Z, 128 (z+1) / Z) and finishes those rows.
// Keeping A in tensor memory leaves shared memory to the TMA ring and its bandwidth
// to the B reads.  B uses the canonical 128-byte-swizzle K-major layout: 8-row atoms
// of 8 x 128 bytes (stride byte offset 1024), the 16-byte chunk of row r at chunk
// index XOR (r mod 8); a K = 32 instruction starts 32 bytes further into its
// 128-column slab.  Every integer sum is exact (|sum| <= 2^20 for K <= 8192).  Every
// wait on an mbarrier is bounded: one that runs out sets status bit 65536 and the
// roles fall through to the common exit; the one cluster barrier (every CTA arrives at
// the start and waits before its sends) is reached by every CTA.

constexpr int kTcWarps = 12;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcEpiThreads = 256;              // warps 0..7
constexpr int kTcLoraThreads = 192;             // warps 6..11
constexpr int kTcM = 128;                       // projection rows per CTA (one UMMA M tile)
constexpr int kTcTiles = kTcM / kTileRows;      // 8 sign tiles per CTA
constexpr int kTcMaxStages = 6;
constexpr int kTcABufs = 4;                     // A buffers in tensor memory
constexpr int kTcACol = 256;                    // first TMEM column of the A buffers
constexpr int kTcTmemCols = 512;
constexpr int kTcMaxSplit = 8;                  // CTAs of one cluster sharing K
constexpr long long kTcSpinLimit = 1LL << 24;
constexpr size_t kTcSmemCap = 225 * 1024;

__host__ __device__ constexpr int tc_stage_bytes(int bg) {
  return 2 * (kDigits * bg) * 128 + kTcTiles * kTileWords * 4;
}
// LoRA sums [128][BG + 1] fp64, the digit-sum terms [BG] int64, the K-split partial
// scaffold sums [128][BG] int64 (the cluster's CTAs x this CTA's rows), alignment slack.
__host__ __device__ constexpr size_t tc_tail_bytes(int bg) {
  return size_t(8) * kTcM * (bg + 1) + size_t(8) * bg + size_t(8) * kTcM * bg + 1024 + 16;
}
// Stages of the TMA ring that fit (at least 2).
__host__ __device__ constexpr int tc_stages(int bg) {
  return (long long)(kTcSmemCap - tc_tail_bytes(bg)) / tc_stage_bytes(bg) > kTcMaxStages
             ? kTcMaxStages
             : int((long long)(kTcSmemCap - tc_tail_bytes(bg)) / tc_stage_bytes(bg));
}
__host__ __device__ constexpr size_t proj_tc_smem_bytes(int bg) {
  return size_t(tc_stages(bg)) * tc_stage_bytes(bg) + tc_tail_bytes(bg);
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: start address, leading
// byte offset 16 (unused by this layout), stride byte offset 1024, version 1.
DFSSM_DEV uint64_t umma_desc_sw128(uint32_t saddr) {
  return uint64_t((saddr >> 4) & 0x3fffu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor of kind::i8: D s32 (c_format 2), A and B both signed 8-bit
// (format 1; the 0/1 sign bytes are valid s8 values, and A and B keep one type),
// both K-major, N >> 3, M = 128 >> 4.
template <int N>
DFSSM_DEV constexpr uint32_t umma_idesc_s8() {
  return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(kTcM >> 4) << 24);
}

DFSSM_DEV void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}

DFSSM_DEV bool tc_wait(uint64_t* bar, unsigned parity, unsigned* status, int* fail) {
  long long spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if (++spins > kTcSpinLimit || *reinterpret_cast<volatile int*>(fail)) {
      if (spins > kTcSpinLimit && status) atomicOr(status, 65536u);
      *reinterpret_cast<volatile int*>(fail) = 1;
      return false;
    }
  }
  return true;
}

DFSSM_DEV void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

// 48 accumulator columns (one batch-row octet) of this warp's 32 TMEM lanes.
DFSSM_DEV void tc_load48(uint32_t taddr, uint32_t (&q)[48]) {
#pragma unroll
  for (int j = 0; j < 3; ++j)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(q[16 * j + 0]), "=r"(q[16 * j + 1]), "=r"(q[16 * j + 2]), "=r"(q[16 * j + 3]),
          "=r"(q[16 * j + 4]), "=r"(q[16 * j + 5]), "=r"(q[16 * j + 6]), "=r"(q[16 * j + 7]),
          "=r"(q[16 * j + 8]), "=r"(q[16 * j + 9]), "=r"(q[16 * j + 10]), "=r"(q[16 * j + 11]),
          "=r"(q[16 * j + 12]), "=r"(q[16 * j + 13]), "=r"(q[16 * j + 14]), "=r"(q[16 * j + 15])
        : "r"(taddr + uint32_t(16 * j)));
}

// Finish one (row, batch-row octet) from its 48 plane sums: sum_d 256^d (2 q_d - T_d)
// is exact in int64 (|q_d| <= 2^20, so q_4 + 256 q_5 fits 32 bits); al 2^-24 is exact,
// so al2 * S rounds once, as al * (S 2^-24) does; then the LoRA term and the store.
template <int EPI, int BG>
DFSSM_DEV void tc_finish(const ProjArgs& a, const uint32_t (&q)[48], int o, int g8, int nb, int b0, double al2,
                         double sb, const long long* Ts, const double* lrow) {
  int bs[8];
  double ys[8];
#pragma unroll
  for (int bi = 0; bi < 8; ++bi) {
    const int* qd = reinterpret_cast<const int*>(&q[bi * kDigits]);
    const long long sq = (long long)qd[0] + (long long)qd[1] * 256 + (long long)qd[2] * 65536 +
                         (long long)qd[3] * 16777216 + (long long)(qd[4] + qd[5] * 256) * 4294967296LL;
    double y = al2 * double(2 * sq - Ts[g8 + bi]);
    if (a.rank > 0) y = fma(sb, lrow[g8 + bi], y);
    bs[bi] = b0 + g8 + bi;
    ys[bi] = y;
  }
  proj_epilogue_group<EPI, 8>(a, o, bs, ys, min(8, nb - g8));
}

template <int EPI, int BG>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_proj_tc(ProjArgs a, const __grid_constant__ CUtensorMap tm_bits, const __grid_constant__ CUtensorMap tm_planes) {
  constexpr int N = kDigits * BG, B_SLAB = N * 128, BITS = kTcTiles * kTileWords * 4;
  constexpr int STAGE = tc_stage_bytes(BG), S = tc_stages(BG), LS = BG + 1;
  static_assert(N % 16 == 0 && N <= kTcACol, "UMMA N and the accumulator columns");
  static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(S >= 2, "two stages at least");
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[kTcMaxStages], empty[kTcMaxStages], aready[kTcABufs], aempty[kTcABufs];
  __shared__ __align__(8) uint64_t done, rbar;
  __shared__ uint32_t tmem_s;
  __shared__ int fail;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kTcM, b0 = blockIdx.y * BG;
  const int ks = gridDim.z, kz = blockIdx.z;                 // K split: cluster (1, 1, ks)
  const int kpc = a.K / kTileCols / ks, kb0 = kz * kpc;      // k-blocks of this CTA
  const int nb = min(BG, a.batch - b0);
  const int LR = kTcM / ks, lr0 = kz * LR;                   // rows this CTA finishes
  const uint32_t raw = smem_u32(smem_raw);
  unsigned char* stages = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(stages);
  double* Ls = reinterpret_cast<double*>(stages + S * STAGE);           // [128][BG + 1] LoRA sums
  long long* Ts = reinterpret_cast<long long*>(Ls + kTcM * LS);         // [BG]: sum_d 256^d T[d]
  long long* rcv = reinterpret_cast<long long*>(                        // [ks][LR][BG] K-split partials
      (reinterpret_cast<uintptr_t>(Ts + BG) + 15) & ~uintptr_t(15));

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(&tmem_s)), "n"(kTcTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 32) {
    for (int i = 0; i < kTcMaxStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kTcABufs; ++i) {
      mbar_init(&aready[i], 4);
      mbar_init(&aempty[i], 1);
    }
    mbar_init(&done, 1);
    mbar_init(&rbar, 1);
    fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_s;
  // the first stages' sign words are weights: requested before the previous kernel
  // (which writes the digit planes, u and the digit sums) has finished
  const int pre = min(S, kpc);
  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tm_bits)) : "memory");
    asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(&tm_planes)) : "memory");
    for (int kb = 0; kb < pre; ++kb) {
      mbar_expect_tx_only(&full[kb], BITS);
      tma_load_2d(sbase + kb * STAGE + 2 * B_SLAB, &tm_bits, (kb0 + kb) * kTileWords, m0 / kTileRows, &full[kb]);
    }
  }
  pdl_wait();
  pdl_release();
  if (ks > 1) {
    // the cluster's barriers are initialised before any CTA sends (the matching
    // wait comes just before the sends); rbar expects every CTA's partials
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    if (tid == 0) mbar_expect_tx(&rbar, unsigned(ks * LR * BG * 8));
  }

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < kpc; ++kb) {
        const int st = kb % S, kg = kb0 + kb;
        if (kb >= S && !tc_wait(&empty[st], unsigned(kb / S - 1) & 1u, a.status, &fail)) break;
        const uint32_t sg = sbase + st * STAGE;
        if (kb < pre) {          // sign words already requested: the planes complete the phase
          mbar_expect_tx(&full[st], 2 * B_SLAB);
        } else {
          mbar_expect_tx(&full[st], BITS + 2 * B_SLAB);
          tma_load_2d(sg + 2 * B_SLAB, &tm_bits, kg * kTileWords, m0 / kTileRows, &full[st]);
        }
        tma_load_2d(sg, &tm_planes, kg * kTileCols, b0 * kDigits, &full[st]);
        tma_load_2d(sg + B_SLAB, &tm_planes, kg * kTileCols + 128, b0 * kDigits, &full[st]);
        issued = kb + 1;
      }
      // no copy may still be landing when the stages are reused or the CTA leaves
      for (int kb = max(0, issued - S); kb < issued; ++kb) {
        long long spins = 0;
        while (!mbar_try_wait(&full[kb % S], unsigned(kb / S) & 1u) && ++spins < kTcSpinLimit) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_s8<N>();
      for (int kb = 0; kb < kpc; ++kb) {
        const int st = kb % S, ab = kb % kTcABufs;
        if (!tc_wait(&full[st], unsigned(kb / S) & 1u, a.status, &fail) ||
            !tc_wait(&aready[ab], unsigned(kb / kTcABufs) & 1u, a.status, &fail))
          break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t bs = sbase + st * STAGE;
        const uint32_t ta = tmem + uint32_t(kTcACol + 64 * ab);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = umma_desc_sw128(bs + (kk >> 2) * B_SLAB + (kk & 3) * 32);
          const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
          asm volatile(
              "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
              " tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n"
              :: "r"(tmem), "r"(ta + 8 * kk), "l"(bd), "r"(idesc), "r"(acc) : "memory");
        }
        tc_commit(&empty[st]);
        tc_commit(&aempty[ab]);
      }
      tc_commit(&done);   // tracks every MMA issued above (also after a wait gave up)
    }
    __syncwarp();
  } else if (warp < 6) {
    // expander: thread = tile row r (TMEM lane).  Row r = 16 tt + 8 hf + g of tile tt
    // lives in the 16-byte words of lanes 4 g + t (t = 0..3): word hf holds, for
    // m = 0..3, bits 2 m (+ 8 i) of columns 64 m + 16 t + i (i = 0..3) and bits 2 m + 1
    // of columns 64 m + 16 t + 8 + i; word hf + 2 the next four columns of each.  The
    // 16-byte K chunk c = 4 m + t of the row is then
    // {w_hf >> 2m, w_hf+2 >> 2m, w_hf >> 2m+1, w_hf+2 >> 2m+1} & 0x01010101.
    const int r = 32 * (warp & 3) + lane, tt = r >> 4, hf = (r >> 3) & 1, g = r & 7;
    const uint32_t trow = tmem + (uint32_t(32 * (warp & 3)) << 16);
    for (int kb = 0; kb < kpc; ++kb) {
      const int st = kb % S, ab = kb % kTcABufs;
      if (kb >= kTcABufs && !tc_wait(&aempty[ab], unsigned(kb / kTcABufs - 1) & 1u, a.status, &fail)) break;
      if (!tc_wait(&full[st], unsigned(kb / S) & 1u, a.status, &fail)) break;
      const unsigned char* wb = stages + st * STAGE + 2 * B_SLAB + tt * 512 + g * 64;
      uint32_t w0[4], w1[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint4 v = *reinterpret_cast<const uint4*>(wb + 16 * t);
        w0[t] = hf ? v.y : v.x;
        w1[t] = hf ? v.w : v.z;
      }
      uint32_t o[64];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int m = c >> 2, t = c & 3;
        o[4 * c + 0] = (w0[t] >> (2 * m)) & 0x01010101u;
        o[4 * c + 1] = (w1[t] >> (2 * m)) & 0x01010101u;
        o[4 * c + 2] = (w0[t] >> (2 * m + 1)) & 0x01010101u;
        o[4 * c + 3] = (w1[t] >> (2 * m + 1)) & 0x01010101u;
      }
      asm volatile(
          "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
          "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,"
          "%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};"
          :: "r"(trow + uint32_t(kTcACol + 64 * ab)),
             "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7]),
             "r"(o[8]), "r"(o[9]), "r"(o[10]), "r"(o[11]), "r"(o[12]), "r"(o[13]), "r"(o[14]), "r"(o[15]),
             "r"(o[16]), "r"(o[17]), "r"(o[18]), "r"(o[19]), "r"(o[20]), "r"(o[21]), "r"(o[22]), "r"(o[23]),
             "r"(o[24]), "r"(o[25]), "r"(o[26]), "r"(o[27]), "r"(o[28]), "r"(o[29]), "r"(o[30]), "r"(o[31]),
             "r"(o[32]), "r"(o[33]), "r"(o[34]), "r"(o[35]), "r"(o[36]), "r"(o[37]), "r"(o[38]), "r"(o[39]),
             "r"(o[40]), "r"(o[41]), "r"(o[42]), "r"(o[43]), "r"(o[44]), "r"(o[45]), "r"(o[46]), "r"(o[47]),
             "r"(o[48]), "r"(o[49]), "r"(o[50]), "r"(o[51]), "r"(o[52]), "r"(o[53]), "r"(o[54]), "r"(o[55]),
             "r"(o[56]), "r"(o[57]), "r"(o[58]), "r"(o[59]), "r"(o[60]), "r"(o[61]), "r"(o[62]), "r"(o[63])
          : "memory");
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&aready[ab]);
    }
  }
  if (warp >= 6) {
    // LoRA stage 2 of rows [lr0, lr0 + LR) on the fp64 tensor cores: L = B_q u^T as
    // m16n8k4 MMAs (rows x batch rows x ranks).  In k-step 4 G + s the fragment column
    // t (thread t of a quad) stands for rank 16 G + 4 t + s, for A (B_q bytes, four
    // ranks per 32-bit load) and B (u, four ranks per two 16-byte loads) alike.
    const int lw = warp - 6, g = lane >> 2, t = lane & 3;
    for (int i = tid - 192; i < BG; i += kTcLoraThreads) {
      long long sum = 0;
      if (i < nb)
        for (int d = kDigits - 1; d >= 0; --d) sum = sum * 256 + a.xdsum[size_t(b0 + i) * kDigits + d];
      Ts[i] = sum;
    }
    const int MT = LR / 16, NT = BG / 8;
    for (int item = lw; item < MT * NT && a.rank > 0; item += kTcLoraThreads / 32) {
      const int mt = lr0 / 16 + item / NT, nt = item % NT;
      const int r0 = 16 * mt + g, r1 = r0 + 8, o0 = m0 + r0, o1 = m0 + r1, bq = b0 + 8 * nt + g;
      double c[4] = {0.0, 0.0, 0.0, 0.0};
      for (int G = 0; G < (a.rank + 15) / 16; ++G) {
        const int j = 16 * G + 4 * t;                      // rank % 4 == 0: j < rank covers j .. j + 3
        const bool jv = j < a.rank;
        const int w0 = (jv && o0 < a.rows) ? __ldg(reinterpret_cast<const int*>(a.B + size_t(o0) * a.rank + j)) : 0;
        const int w1 = (jv && o1 < a.rows) ? __ldg(reinterpret_cast<const int*>(a.B + size_t(o1) * a.rank + j)) : 0;
        double2 ua = make_double2(0.0, 0.0), ub = ua;
        if (jv && 8 * nt + g < nb) {
          const double2* up = reinterpret_cast<const double2*>(a.u + size_t(bq) * a.rank + j);
          ua = up[0];
          ub = up[1];
        }
        const double uv[4] = {ua.x, ua.y, ub.x, ub.y};
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          const double a0 = double(int8_t(w0 >> (8 * s4))), a1 = double(int8_t(w1 >> (8 * s4)));
          asm volatile("mma.sync.aligned.m16n8k4.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
                       : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3]) : "d"(a0), "d"(a1), "d"(uv[s4]));
        }
      }
      // D fragment: (r0, 2t), (r0, 2t + 1), (r1, 2t), (r1, 2t + 1) of the 16 x 8 tile
      Ls[r0 * LS + 8 * nt + 2 * t] = c[0];
      Ls[r0 * LS + 8 * nt + 2 * t + 1] = c[1];
      Ls[r1 * LS + 8 * nt + 2 * t] = c[2];
      Ls[r1 * LS + 8 * nt + 2 * t + 1] = c[3];
    }
  }
  // the epilogue warps wait for the MMAs; everyone then sees Ls and Ts
  bool ok = true;
  if (warp < 8) {
    ok = tc_wait(&done, 0u, a.status, &fail);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  }
  __syncthreads();
  ok = ok && !*reinterpret_cast<volatile int*>(&fail);
  const int quarter = warp & 3, h = (warp >> 2) & 1;
  if (ks == 1) {
    if (warp < 8) {
      // warp w: TMEM lanes 32 (w mod 4) .. + 31, batch-row octets w / 4, + 2, ...
      const int r = 32 * quarter + lane, o = m0 + r;
      const double al2 = o < a.rows ? h2d(a.alpha[o]) * (1.0 / 16777216.0) : 0.0;
      const double sb = (o < a.rows && a.rank > 0) ? h2d(a.sB[o]) : 0.0;
      for (int g8 = 8 * h; g8 < BG; g8 += 16) {
        uint32_t q[48];
        tc_load48(tmem + (uint32_t(32 * quarter) << 16) + uint32_t(g8 * kDigits), q);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (ok && o < a.rows) tc_finish<EPI, BG>(a, q, o, g8, nb, b0, al2, sb, Ts, Ls + r * LS);
      }
    }
  } else {
    // K split: each epilogue thread folds its row's plane sums into one exact int64
    // partial sum_d 256^d q_d per batch row and stores it (st.async) into the CTA
    // that finishes the row, slot [kz][row - its first row][batch row]; that CTA adds
    // the cluster's partials once its barrier has counted all of them
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (warp < 8) {
      const int r = 32 * quarter + lane, p = r / LR, rl = r % LR;
      const uint32_t dst = cluster_map(smem_u32(rcv + (kz * LR + rl) * BG), unsigned(p));
      const uint32_t bar = cluster_map(smem_u32(&rbar), unsigned(p));
      for (int g8 = 8 * h; g8 < BG; g8 += 16) {
        uint32_t q[48];
        tc_load48(tmem + (uint32_t(32 * quarter) << 16) + uint32_t(g8 * kDigits), q);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int bi = 0; bi < 8; bi += 2) {
          long long sq[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int* qd = reinterpret_cast<const int*>(&q[(bi + e) * kDigits]);
            sq[e] = (long long)qd[0] + (long long)qd[1] * 256 + (long long)qd[2] * 65536 +
                    (long long)qd[3] * 16777216 + (long long)(qd[4] + qd[5] * 256) * 4294967296LL;
          }
          asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.s64 [%0], {%1, %2}, [%3];"
                       :: "r"(dst + uint32_t(8 * (g8 + bi))), "l"(sq[0]), "l"(sq[1]), "r"(bar) : "memory");
        }
      }
    }
    if (tid < kTcEpiThreads) {
      const bool got = tc_wait(&rbar, 0u, a.status, &fail);
      const int rl = tid % LR, slot = tid / LR, nslot = kTcEpiThreads / LR;
      const int r = lr0 + rl, o = m0 + r;
      const double al2 = o < a.rows ? h2d(a.alpha[o]) * (1.0 / 16777216.0) : 0.0;
      const double sb = (o < a.rows && a.rank > 0) ? h2d(a.sB[o]) : 0.0;
      // batch rows slot, slot + nslot, ... (at most 8: nslot >= 4 as LR <= 64)
      int bs[8];
      double ys[8];
      int n = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int b8 = slot + i * nslot;
        bs[i] = b0 + b8;
        ys[i] = 0.0;
        if (b8 < BG && b8 < nb) {
          long long sq = 0;
          for (int p = 0; p < ks; ++p) sq += rcv[(p * LR + rl) * BG + b8];
          double y = al2 * double(2 * sq - Ts[b8]);
          if (a.rank > 0) y = fma(sb, Ls[r * LS + b8], y);
          ys[i] = y;
          n = i + 1;
        }
      }
      if (got && ok && o < a.rows) proj_epilogue_group<EPI, 8>(a, o, bs, ys, n);
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "n"(kTcTmemCols) : "memory");
}

// ------------------------------------------------------------------ SSM step

struct SsmArgs {
  int H, P, N, E, conv_dim, in_rows;
  const double* zx;      // fp64 [B][in_rows]
  const double* xc;      // fp64 [B][conv_dim]
  const float* dt_bias;
  const float* A_log;
  const float* D;
  void* state;           // [B][H][P][N], fp32 or (state16) fp16
  bool state16;
  float* g;              // fp32 [B][E]
  int dt_lo;             // zx row of head 0's raw step size (rows dt_lo .. dt_lo + H - 1)
  int batch;
  unsigned* status;      // value 32768 is or-ed in if a streamed copy did not land (k_ssm_stream)
};

constexpr int kSsmThreads = 256;

// Step size and decay of (batch row b, head h) from the in_proj output:
// dt = softplus(dt_raw + dt_bias), dA = exp(-dt exp(A_log)), in fp64.
DFSSM_DEV double2 step_and_decay(const SsmArgs& a, int b, int h) {
  const double dt = softplus_d(a.zx[size_t(b) * a.in_rows + a.dt_lo + h] + double(a.dt_bias[h]));
  return make_double2(dt, exp(dt * -exp(double(a.A_log[h]))));
}

// Sum over the warp of R per-lane values, folded so that each shuffle level halves
// the values a lane carries: afterwards every lane holds the full sum of value
// `*sel` (lanes that differ only in their low bits hold the same one).
template <int R>
DFSSM_DEV double fold_rows(double (&y)[R], int lane, int* sel) {
  int s = 0, off = 16;
#pragma unroll
  for (int n = R; n > 1; n >>= 1, off >>= 1) {
    const bool hi = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const double keep = hi ? y[j + n / 2] : y[j];
      const double send = hi ? y[j] : y[j + n / 2];
      y[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
    s = 2 * s + (hi ? 1 : 0);
  }
  double v = y[0];
  for (; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  *sel = s;
  return v;
}

// grid (H, B): one block per head and batch row; warp w owns state rows w, w + 8, ...
// A lane holds NCH float4 of a row (columns 4 (lane + 32 c)), and a warp keeps
// 8 / NCH rows in flight: their state loads are issued before anything else (they
// depend on nothing), then B, C, x and the step size and decay arrive (computed from
// the raw step-size row: dt = softplus(dt_raw + dt_bias), dA = exp(-dt * exp(A_log))).
// Arithmetic in fp64, state stored back in fp32 with
// streaming hints (read and written once per step):
//   h' = dA h + (x dt) B,  y = C . h' + D x,  g = y * silu(z) (stored fp32).
// Four consecutive state values (16-byte aligned for fp32, 8-byte for fp16) as
// floats, with a streaming hint; and four fp64 updates stored back, rounded once to
// the state's type.
DFSSM_DEV float4 ld_state4(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
DFSSM_DEV float4 ld_state4(const __half* p) {
  const uint2 v = __ldcs(reinterpret_cast<const uint2*>(p));
  return make_float4(h2f(uint16_t(v.x & 0xffffu)), h2f(uint16_t(v.x >> 16)), h2f(uint16_t(v.y & 0xffffu)),
                     h2f(uint16_t(v.y >> 16)));
}
DFSSM_DEV void st_state4(float* p, double h0, double h1, double h2, double h3) {
  __stcs(reinterpret_cast<float4*>(p), make_float4(float(h0), float(h1), float(h2), float(h3)));
}
DFSSM_DEV void st_state4(__half* p, double h0, double h1, double h2, double h3) {
  const uint2 v = make_uint2(uint32_t(d2h(h0)) | (uint32_t(d2h(h1)) << 16),
                             uint32_t(d2h(h2)) | (uint32_t(d2h(h3)) << 16));
  __stcs(reinterpret_cast<uint2*>(p), v);
}

template <int NCH, typename ST>
__global__ void __launch_bounds__(kSsmThreads, 2) k_ssm(SsmArgs a) {
  constexpr int RW = 8 / NCH;                  // rows of a warp in flight
  constexpr int kW = kSsmThreads / 32;
  const int h = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N4 = a.N / 4, P = a.P;
  ST* sbase = static_cast<ST*>(a.state) + (size_t(b) * a.H + h) * size_t(P) * a.N;
  const double* xcb = a.xc + size_t(b) * a.conv_dim;
  const double* zr = a.zx + size_t(b) * a.in_rows;
  for (int r0 = warp; r0 < P; r0 += RW * kW) {
    float4 hv[RW][NCH];
#pragma unroll
    for (int i = 0; i < RW; ++i)
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int p = r0 + i * kW, n4 = lane + 32 * c;
        hv[i][c] = (p < P && n4 < N4) ? ld_state4(sbase + size_t(p) * a.N + 4 * n4)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    pdl_wait();                            // B, C, x, z and dt come from the in_proj
    pdl_release();
    double Bv[NCH][4], Cv[NCH][4];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int n4 = lane + 32 * c;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        Bv[c][e] = n4 < N4 ? xcb[a.E + 4 * n4 + e] : 0.0;
        Cv[c][e] = n4 < N4 ? xcb[a.E + a.N + 4 * n4 + e] : 0.0;
      }
    }
    double xv[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) xv[i] = r0 + i * kW < P ? xcb[h * P + r0 + i * kW] : 0.0;
    const double2 sd = step_and_decay(a, b, h);
    const double dt = sd.x, dA = sd.y;
    double y[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      const double xdt = xv[i] * dt;
      const int p = r0 + i * kW;
      double acc = 0.0;
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int n4 = lane + 32 * c;
        const double h0 = fma(dA, double(hv[i][c].x), xdt * Bv[c][0]);
        const double h1 = fma(dA, double(hv[i][c].y), xdt * Bv[c][1]);
        const double h2 = fma(dA, double(hv[i][c].z), xdt * Bv[c][2]);
        const double h3 = fma(dA, double(hv[i][c].w), xdt * Bv[c][3]);
        acc = fma(Cv[c][0], h0, acc);
        acc = fma(Cv[c][1], h1, acc);
        acc = fma(Cv[c][2], h2, acc);
        acc = fma(Cv[c][3], h3, acc);
        if (p < P && n4 < N4) st_state4(sbase + size_t(p) * a.N + 4 * n4, h0, h1, h2, h3);
      }
      y[i] = acc;
    }
    int sel;
    const double ys = fold_rows<RW>(y, lane, &sel);
    // lanes 0, 32/RW, ... hold distinct rows
    const int p = r0 + sel * kW;
    if ((lane & (32 / RW - 1)) == 0 && p < P) {
      const int e = h * P + p;
      const double yy = fma(double(a.D[h]), xcb[e], ys);
      a.g[size_t(b) * a.E + e] = float(yy * silu_d(zr[e]));
    }
  }
}

// k_ssm_stream items: (batch row, head, part), the part being P / kSsmSplit state
// rows (rows update independently given B, C, x and the step size).  Bytes of an item
// and their offsets in a buffer: state [RP][N] (es bytes per value), then B and C
// [2N] fp64, x [RP] fp64, z [RP] fp64.
#ifndef DFSSM_SSM_SPLIT
#define DFSSM_SSM_SPLIT 1
#endif
#ifndef DFSSM_SSM_BUFS
#define DFSSM_SSM_BUFS 2
#endif
// Measured at batch 64 (ms per 48-layer step): whole items with 2 buffers 4.92;
// halves with 2 / 3 / 4 buffers 5.29 / 5.43 / 6.07; quarters with 4 buffers 7.37 -- the
// per-item fixed work (B and C into registers, two block barriers, the row folds), not
// the bytes in flight, is what smaller items add.
constexpr int kSsmSplit = DFSSM_SSM_SPLIT;   // parts per (batch, head)
constexpr int kSsmBufs = DFSSM_SSM_BUFS;     // shared-memory buffers per block
struct SsmItem {
  int rows, st, bc, x, z, bytes;
};
__host__ __device__ inline SsmItem ssm_item(int P, int N, int es) {
  SsmItem it;
  it.rows = P / kSsmSplit;
  it.st = 0;
  it.bc = ((es * it.rows * N + 15) / 16) * 16;
  it.x = it.bc + 16 * N;
  it.z = it.x + 8 * it.rows;
  it.bytes = it.z + 8 * it.rows;
  return it;
}
constexpr int kSsmStreamThreads = 256;
constexpr int kSsmStreamMaxItems = 256;   // items per block (a step-size table entry each)

// Streaming SSM update: grid of resident blocks; block c takes the items c,
// c + gridDim.x, ... (at most kSsmStreamMaxItems).  Each item's inputs (its RP N
// values of state, the batch row's B and C, the rows' x and z) arrive by bulk copies
// into one of kSsmBufs shared-memory buffers; a buffer is refilled with the item
// kSsmBufs further on as soon as its item is computed, so a block keeps kSsmBufs - 1
// items in flight while it computes one.  The block's step sizes and decays are
// computed up front, one item per thread, while the first copies land.  Warp w takes
// rows w, w + 8, ... four at a time; a lane holds NCH float4 of a row.  Same
// arithmetic as k_ssm (fp64, state stored back in its own type with a streaming hint).
// Four consecutive state values from shared memory, converted once to fp64 (fp16
// goes straight to fp64: one exact conversion per value).
struct D4 {
  double x, y, z, w;
};
DFSSM_DEV double h2d_direct(uint16_t h) {
  double r;
  asm("cvt.f64.f16 %0, %1;" : "=d"(r) : "h"(h));
  return r;
}
DFSSM_DEV D4 ld_smem_state4(const float* p) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  return D4{double(v.x), double(v.y), double(v.z), double(v.w)};
}
DFSSM_DEV D4 ld_smem_state4(const __half* p) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  return D4{h2d_direct(uint16_t(v.x & 0xffffu)), h2d_direct(uint16_t(v.x >> 16)),
            h2d_direct(uint16_t(v.y & 0xffffu)), h2d_direct(uint16_t(v.y >> 16))};
}

template <int NCH, typename ST>
__global__ void __launch_bounds__(kSsmStreamThreads) k_ssm_stream(SsmArgs a) {
  extern __shared__ __align__(16) unsigned char sbuf[];
  __shared__ __align__(8) uint64_t bar[kSsmBufs];
  __shared__ int s_ok;
  __shared__ double2 sdt[kSsmStreamMaxItems];
  constexpr int RW = 4, kW = kSsmStreamThreads / 32;
  const int P = a.P, N = a.N, H = a.H, N4 = N / 4;
  const SsmItem it = ssm_item(P, N, int(sizeof(ST)));
  const int RP = it.rows;
  const int bufb = (it.bytes + 127) & ~127;
  const int nitems = a.batch * H * kSsmSplit;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int j = 0; j < kSsmBufs; ++j) mbar_init(&bar[j], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  int issued[kSsmBufs], landed[kSsmBufs];   // thread 0: copy phases per buffer
#pragma unroll
  for (int j = 0; j < kSsmBufs; ++j) issued[j] = landed[j] = 0;
  // an item's copies: its state (written only by this kernel, so it may be requested
  // before the previous kernel has finished), then B, C, x and z (the in_proj output)
  auto issue_state = [&](int item, int buf) {
    ++issued[buf];
    const int bh = item / kSsmSplit, part = item % kSsmSplit, b = bh / H, h = bh % H, r0 = part * RP;
    mbar_expect_tx(&bar[buf], unsigned(it.bytes));
    bulk_g2s(sbuf + buf * bufb + it.st, static_cast<const ST*>(a.state) + ((size_t(b) * H + h) * P + r0) * N,
             unsigned(sizeof(ST) * RP * N), &bar[buf]);
  };
  auto issue_inputs = [&](int item, int buf) {
    const int bh = item / kSsmSplit, part = item % kSsmSplit, b = bh / H, h = bh % H, r0 = part * RP;
    unsigned char* base = sbuf + buf * bufb;
    bulk_g2s(base + it.bc, a.xc + size_t(b) * a.conv_dim + a.E, unsigned(16 * N), &bar[buf]);
    bulk_g2s(base + it.x, a.xc + size_t(b) * a.conv_dim + size_t(h) * P + r0, unsigned(8 * RP), &bar[buf]);
    bulk_g2s(base + it.z, a.zx + size_t(b) * a.in_rows + size_t(h) * P + r0, unsigned(8 * RP), &bar[buf]);
  };
  auto issue = [&](int item, int buf) {
    issue_state(item, buf);
    issue_inputs(item, buf);
  };
  if (tid == 0)
    for (int j = 0; j < kSsmBufs; ++j)
      if (int(blockIdx.x + j * gridDim.x) < nitems) issue_state(blockIdx.x + j * gridDim.x, j);
  pdl_wait();
  pdl_release();
  if (tid == 0)
    for (int j = 0; j < kSsmBufs; ++j)
      if (int(blockIdx.x + j * gridDim.x) < nitems) issue_inputs(blockIdx.x + j * gridDim.x, j);
  for (int k = tid; k < kSsmStreamMaxItems; k += kSsmStreamThreads) {
    const int item = int(blockIdx.x) + k * int(gridDim.x);
    if (item < nitems) {
      const int bh = item / kSsmSplit;
      sdt[k] = step_and_decay(a, bh / H, bh % H);
    }
  }
  for (int k = 0;; ++k) {
    const int item = int(blockIdx.x) + k * int(gridDim.x);
    if (item >= nitems) break;
    const int buf = k % kSsmBufs;
    const unsigned par = unsigned(k / kSsmBufs) & 1u;
    if (tid == 0) {
      long long spins = 0;
      bool ok = true;
      while (!mbar_try_wait(&bar[buf], par))
        if (++spins > (1 << 22)) { ok = false; break; }
      s_ok = ok ? 1 : 0;
      if (ok) {
        ++landed[buf];
      } else {
        atomicOr(a.status, 32768u);
        // Before the block exits, let every copy still in flight towards its shared
        // memory land: each buffer has at most one outstanding phase, whose parity is
        // that of its last issue (bounded again; the status already marks the outputs
        // invalid).
        for (int bb = 0; bb < kSsmBufs; ++bb) {
          if (issued[bb] == landed[bb]) continue;
          const unsigned pp = unsigned(issued[bb] - 1) & 1u;
          long long s2 = 0;
          while (!mbar_try_wait(&bar[bb], pp) && ++s2 < (1LL << 24)) __nanosleep(64);
        }
      }
    }
    __syncthreads();
    if (!s_ok) return;
    (void)mbar_try_wait(&bar[buf], par);   // every thread acquires the copies' writes
    const unsigned char* base = sbuf + buf * bufb;
    const ST* st = reinterpret_cast<const ST*>(base + it.st);
    const double* Bs = reinterpret_cast<const double*>(base + it.bc);
    const double* Cs = Bs + N;
    const double* xs = reinterpret_cast<const double*>(base + it.x);
    const double* zs = reinterpret_cast<const double*>(base + it.z);
    const double dt = sdt[k].x, dA = sdt[k].y;
    const int bh = item / kSsmSplit, b = bh / H, h = bh % H, rbase = (item % kSsmSplit) * RP;
    ST* gst = static_cast<ST*>(a.state) + ((size_t(b) * H + h) * P + rbase) * N;
    double Bv[NCH][4], Cv[NCH][4];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int n4 = lane + 32 * c;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        Bv[c][e] = n4 < N4 ? Bs[4 * n4 + e] : 0.0;
        Cv[c][e] = n4 < N4 ? Cs[4 * n4 + e] : 0.0;
      }
    }
    for (int r0 = warp; r0 < RP; r0 += RW * kW) {
      double y[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int p = r0 + i * kW;
        const double xdt = p < RP ? xs[p] * dt : 0.0;
        double acc = 0.0;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          const int n4 = lane + 32 * c;
          if (p < RP && n4 < N4) {
            const D4 hv = ld_smem_state4(st + size_t(p) * N + 4 * n4);
            const double h0 = fma(dA, hv.x, xdt * Bv[c][0]);
            const double h1 = fma(dA, hv.y, xdt * Bv[c][1]);
            const double h2 = fma(dA, hv.z, xdt * Bv[c][2]);
            const double h3 = fma(dA, hv.w, xdt * Bv[c][3]);
            acc = fma(Cv[c][0], h0, acc);
            acc = fma(Cv[c][1], h1, acc);
            acc = fma(Cv[c][2], h2, acc);
            acc = fma(Cv[c][3], h3, acc);
            st_state4(gst + size_t(p) * N + 4 * n4, h0, h1, h2, h3);
          }
        }
        y[i] = acc;
      }
      int sel;
      const double ys = fold_rows<RW>(y, lane, &sel);
      const int p = r0 + sel * kW;
      if ((lane & (32 / RW - 1)) == 0 && p < RP) {
        const int e = h * P + rbase + p;
        const double yy = fma(double(a.D[h]), xs[p], ys);
        a.g[size_t(b) * a.E + e] = float(yy * silu_d(zs[p]));
      }
    }
    __syncthreads();   // buffer consumed
    if (tid == 0 && item + kSsmBufs * int(gridDim.x) < nitems) issue(item + kSsmBufs * int(gridDim.x), buf);
  }
}

// ------------------------------------------------------------------ density-field state codec
//
// "Density Field State Space Models", Section 3.4 and Appendix D: a state row of n
// values is held as a K x K binary field (K^2 >= 4 n; K = 23 at d_state 128), four
// cells per value in raster order, the spare cells 0.  The row's mean mu and
// population standard deviation sigma (fp64, summed left to right) give
// lo = mu - 3 sigma and span = 6 sigma, kept as fp32; value i's 8-bit code is
// q = rint(255 clip((h - lo) / span, 0, 1)) (128 if span is 0); a first-order
// sigma-delta with a signed 8-bit error e (0 at the row's first cell, carried along
// the row) sets cell = [e + q >= 128] and e <- e + q - 255 cell; the readout is
// lo + span (ones among the value's cells) / 4.  Every fp64 step is an explicitly
// rounded intrinsic in a fixed order (no contraction), so the integer decisions are
// the same as in any other IEEE evaluation of these formulas.

constexpr int kDfCells = 4;   // cells per state value

__host__ __device__ inline int df_field_k(int n) {
  int K = 1;
  while (K * K < kDfCells * n) ++K;
  return K;
}
__host__ __device__ inline int df_field_words(int n) {
  const int K = df_field_k(n);
  return (K * K + 31) / 32;
}

// One row: get(i) reads value i, put(i, v) receives its readout (after get(i) has
// been read for the last time); cells (may be null) receives the field, 32 cells a
// word, low bit first; lo and span are returned.
template <typename Get, typename Put>
DFSSM_DEV void df_row(int n, Get get, Put put, uint32_t* cells, float* lo_out, float* span_out) {
  double total = 0.0;
  for (int i = 0; i < n; ++i) total = __dadd_rn(total, get(i));
  const double mu = __ddiv_rn(total, double(n));
  double ss = 0.0;
  for (int i = 0; i < n; ++i) {
    const double d = __dsub_rn(get(i), mu);
    ss = __dadd_rn(ss, __dmul_rn(d, d));
  }
  const double sigma = __dsqrt_rn(__ddiv_rn(ss, double(n)));
  const float lo = __double2float_rn(__dsub_rn(mu, __dmul_rn(3.0, sigma)));
  const float span = __double2float_rn(__dmul_rn(6.0, sigma));
  const double lod = double(lo), spand = double(span);
  int e = 0;
  uint32_t word = 0u;
  for (int i = 0; i < n; ++i) {
    int q = 128;
    if (span != 0.f) {
      const double t = __ddiv_rn(__dsub_rn(get(i), lod), spand);
      q = int(rint(__dmul_rn(255.0, fmin(1.0, fmax(0.0, t)))));
    }
    int ones = 0;
#pragma unroll
    for (int j = 0; j < kDfCells; ++j) {
      const int sum = e + q;
      const int bit = sum >= 128 ? 1 : 0;
      e = sum - 255 * bit;
      ones += bit;
      const int c = kDfCells * i + j;
      word |= uint32_t(bit) << (c & 31);
      if ((c & 31) == 31) {
        if (cells) cells[c >> 5] = word;
        word = 0u;
      }
    }
    put(i, __dadd_rn(lod, __dmul_rn(double(ones) * (1.0 / kDfCells), spand)));
  }
  if (cells) {
    const int K = df_field_k(n), words = (K * K + 31) / 32;
    int w = (kDfCells * n) >> 5;
    if ((kDfCells * n) & 31) cells[w++] = word;   // the last partial word, spare cells 0
    for (; w < words; ++w) cells[w] = 0u;
  }
  if (lo_out) *lo_out = lo;
  if (span_out) *span_out = span;
}

// grid (ceil(rows / 128)), 128 threads: thread = one row of n fp32 values -> its field
// (words_per_row words), lo and span; rows_out (may be null, may alias rows) gets the
// readout.
__global__ void __launch_bounds__(128) k_df_encode(const float* rows, int n_rows, int n, uint32_t* cells,
                                                    float* lo, float* span, float* rows_out) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= n_rows) return;
  const float* src = rows + size_t(r) * n;
  float* dst = rows_out ? rows_out + size_t(r) * n : nullptr;
  const int words = df_field_words(n);
  df_row(
      n, [&](int i) { return double(src[i]); },
      [&](int i, double v) {
        if (dst) dst[i] = __double2float_rn(v);
      },
      cells + size_t(r) * words, lo + r, span + r);
}

// grid (ceil(rows / 128)), 128 threads: readout of each row's field into fp32.
__global__ void __launch_bounds__(128) k_df_decode(const uint32_t* cells, const float* lo, const float* span,
                                                    int n_rows, int n, float* rows) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= n_rows) return;
  const uint32_t* f = cells + size_t(r) * df_field_words(n);
  const double lod = double(lo[r]), spand = double(span[r]);
  for (int i = 0; i < n; ++i) {
    const int c = kDfCells * i;
    const int ones = __popc((f[c >> 5] >> (c & 31)) & ((1u << kDfCells) - 1u));
    rows[size_t(r) * n + i] = __double2float_rn(__dadd_rn(lod, __dmul_rn(double(ones) * (1.0 / kDfCells), spand)));
  }
}

// ------------------------------------------------------------------ prompt pass (prefill)
//
// A prompt of T tokens per batch row goes through a layer in one pass: the
// projections run on all B*T token rows at once (k_prologue_cl, k_proj), the conv
// runs along the sequence (k_conv_seq) and the selective SSM as the chunked scan of
// Mamba-2's state space duality form ("Density Field State Space Models", Section 2;
// block_len 64 as in Appendix B) in k_ssd.

struct PrefillArgs {
  int B, T, H, P, N, E, C, in_rows;   // batch, prompt length, heads, headdim, d_state, d_inner, conv_dim, in_proj rows
  const double* zx;         // fp64 [B*T][in_rows]: [z | x B C | dt] of every prompt token
  const uint16_t* conv_w;   // fp16 [C][4]
  const uint16_t* conv_b;   // fp16 [C]
  float* conv_state;        // fp32 [B][3][C], in/out
  double* xc;               // fp64 [B*T][C] conv outputs after SiLU
  const float* dt_bias;     // [H]
  const float* A_log;       // [H]
  const float* D;           // [H]
  void* state;              // [B][H][P][N], fp32 or (state16) fp16, in/out
  bool state16;
  float* g;                 // fp32 [B*T][E] gated value y * silu(z)
  bool df;                  // density-field codec on the state carried between chunks (DF-SSD)
};

// grid (ceil(C / 256), B), 256 threads: one thread per conv channel walks the prompt
// with the three stored inputs in registers (the prompt's own inputs enter the
// window at full precision; the state is stored back as fp32 at the end).
__global__ void __launch_bounds__(256) k_conv_seq(PrefillArgs a) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x, b = blockIdx.y;
  if (c >= a.C) return;
  float* cs = a.conv_state + size_t(b) * 3 * a.C;
  double s0 = cs[c], s1 = cs[a.C + c], s2 = cs[2 * a.C + c];
  const uint2 wv = *reinterpret_cast<const uint2*>(a.conv_w + size_t(c) * 4);
  const double w0 = h2d(uint16_t(wv.x & 0xffff)), w1 = h2d(uint16_t(wv.x >> 16));
  const double w2 = h2d(uint16_t(wv.y & 0xffff)), w3 = h2d(uint16_t(wv.y >> 16));
  const double bias = h2d(a.conv_b[c]);
  for (int t = 0; t < a.T; ++t) {
    const size_t row = size_t(b) * a.T + t;
    const double x = a.zx[row * a.in_rows + a.E + c];   // conv rows follow the E z rows
    double pre = bias;
    pre = fma(w0, s0, pre);
    pre = fma(w1, s1, pre);
    pre = fma(w2, s2, pre);
    pre = fma(w3, x, pre);
    a.xc[row * a.C + c] = silu_d(pre);
    s0 = s1;
    s1 = s2;
    s2 = x;
  }
  cs[c] = float(s0);
  cs[a.C + c] = float(s1);
  cs[2 * a.C + c] = float(s2);
}

constexpr int kSsdL = 64;             // chunk length (block_len)
constexpr int kSsdThreads = 256;

// Shared memory of k_ssd: the state (transposed, [N][P] fp64), the chunk's x [L][P]
// fp64, B transposed [N][L] and C [L][N] (fp32 copies of the fp64 conv outputs),
// M [L][L] fp64, and per-token step sizes, cumulative log-decays and weights.
__host__ __device__ inline size_t ssd_smem_bytes(int P, int N) {
  return size_t(8) * P * N + size_t(8) * kSsdL * P + size_t(4) * 2 * kSsdL * N + size_t(8) * kSsdL * kSsdL +
         size_t(8) * 4 * kSsdL;
}

DFSSM_DEV double ld_state(const float* p) { return double(*p); }
DFSSM_DEV double ld_state(const __half* p) { return h2d(__half_as_ushort(*p)); }
DFSSM_DEV void st_state(float* p, double v) { *p = float(v); }
DFSSM_DEV void st_state(__half* p, double v) { *p = __ushort_as_half(d2h(v)); }

// grid (H, B), 256 threads: one CTA per (batch row, head) walks the prompt in chunks
// of up to 64 tokens, the state carried in fp64 in shared memory.  Per chunk, with
// dt_t = softplus(dt_raw_t + dt_bias), cs_t = sum_{r <= t} dt_r A (A = -exp(A_log)):
//   M[t][s] = (C_t . B_s) exp(cs_t - cs_s) dt_s  (s <= t),
//   y_t[p]  = sum_s M[t][s] x_s[p] + exp(cs_t) (C_t . h[p]) + D x_t[p],
//   h[p][n] <- exp(cs_end) h[p][n] + sum_s exp(cs_end - cs_s) dt_s x_s[p] B_s[n],
// and g = y silu(z) is stored in fp32.  The state is read once and written once
// (rounded to its storage type).  With a.df the state carried into each next chunk
// passes through the density-field codec (df_row); the final state does not.
template <typename ST>
__global__ void __launch_bounds__(kSsdThreads) k_ssd(PrefillArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int P = a.P, N = a.N, T = a.T, E = a.E, C = a.C;
  double* hs = reinterpret_cast<double*>(smem);            // [N][P]
  double* xs = hs + P * N;                                  // [L][P]
  float* BsT = reinterpret_cast<float*>(xs + kSsdL * P);    // [N][L]
  float* Cs = BsT + kSsdL * N;                              // [L][N]
  double* M = reinterpret_cast<double*>(Cs + kSsdL * N);    // [L][L]
  double* dts = M + kSsdL * kSsdL;                          // [L]
  double* cs = dts + kSsdL;                                 // [L]
  double* ecs = cs + kSsdL;                                 // [L] exp(cs_t)
  double* wend = ecs + kSsdL;                               // [L] exp(cs_end - cs_s) dt_s
  ST* gst = static_cast<ST*>(a.state) + (size_t(b) * a.H + h) * P * N;
  for (int i = tid; i < P * N; i += blockDim.x) {
    const int p = i / N, n = i % N;
    hs[n * P + p] = ld_state(gst + i);
  }
  const double A = -exp(double(a.A_log[h])), Dh = double(a.D[h]), dtb = double(a.dt_bias[h]);
  for (int c0 = 0; c0 < T; c0 += kSsdL) {
    const int L = min(kSsdL, T - c0);
    __syncthreads();   // the previous chunk is done with the buffers
    for (int i = tid; i < L * P; i += blockDim.x) {
      const int t = i / P, p = i % P;
      xs[i] = a.xc[(size_t(b) * T + c0 + t) * C + h * P + p];
    }
    for (int i = tid; i < L * N; i += blockDim.x) {
      const int t = i / N, n = i % N;
      const double* row = a.xc + (size_t(b) * T + c0 + t) * C + E;
      BsT[n * kSsdL + t] = float(row[n]);
      Cs[t * N + n] = float(row[N + n]);
    }
    if (tid < L)
      dts[tid] = softplus_d(a.zx[(size_t(b) * T + c0 + tid) * a.in_rows + E + C + h] + dtb);
    __syncthreads();
    if (tid == 0) {                 // cumulative log-decay, left to right
      double acc = 0.0;
      for (int t = 0; t < L; ++t) {
        acc += dts[t] * A;
        cs[t] = acc;
      }
    }
    __syncthreads();
    if (tid < L) {
      ecs[tid] = exp(cs[tid]);
      wend[tid] = exp(cs[L - 1] - cs[tid]) * dts[tid];
    }
    for (int i = tid; i < L * L; i += blockDim.x) {
      const int t = i / L, s = i % L;
      double v = 0.0;
      if (s <= t) {
        double cb = 0.0;
        for (int n = 0; n < N; ++n) cb = fma(double(Cs[t * N + n]), double(BsT[n * kSsdL + s]), cb);
        v = cb * exp(cs[t] - cs[s]) * dts[s];
      }
      M[t * kSsdL + s] = v;
    }
    __syncthreads();
    for (int i = tid; i < L * P; i += blockDim.x) {
      const int t = i / P, p = i % P;
      double y = 0.0;
      for (int s = 0; s <= t; ++s) y = fma(M[t * kSsdL + s], xs[s * P + p], y);
      double yi = 0.0;
      for (int n = 0; n < N; ++n) yi = fma(double(Cs[t * N + n]), hs[n * P + p], yi);
      y = fma(ecs[t], yi, y);
      y = fma(Dh, xs[t * P + p], y);
      const size_t row = size_t(b) * T + c0 + t;
      const double z = a.zx[row * a.in_rows + h * P + p];
      a.g[row * E + h * P + p] = float(y * silu_d(z));
    }
    __syncthreads();
    const double eend = exp(cs[L - 1]);
    for (int i = tid; i < P * N; i += blockDim.x) {
      const int n = i / P, p = i % P;
      double acc = 0.0;
      for (int s = 0; s < L; ++s) acc = fma(wend[s] * xs[s * P + p], double(BsT[n * kSsdL + s]), acc);
      hs[i] = fma(eend, hs[i], acc);
    }
    if (a.df && c0 + kSsdL < T) {
      // DF-SSD: the state carried into the next chunk is the density-field readout of
      // this one's (thread p: state row p, column p of hs)
      __syncthreads();
      if (tid < P)
        df_row(
            N, [&](int n) { return hs[n * P + tid]; }, [&](int n, double v) { hs[n * P + tid] = v; }, nullptr,
            nullptr, nullptr);
    }
  }
  __syncthreads();
  for (int i = tid; i < P * N; i += blockDim.x) {
    const int p = i / N, n = i % N;
    st_state(gst + i, hs[n * P + p]);
  }
}

// grid (B), 256 threads: dst[b] = src[b * T + T - 1] (rows of D floats).
__global__ void k_last_rows(const float* __restrict__ src, int T, int D, float* __restrict__ dst) {
  const int b = blockIdx.x;
  for (int k = threadIdx.x; k < D; k += blockDim.x) dst[size_t(b) * D + k] = src[(size_t(b) * T + T - 1) * D + k];
}

// ------------------------------------------------------------------ embedding / LM head

// grid (B).  residual row b = embedding row tok[b]: fp16 as given, or int8 codes times
// the row's fp32 scale (an fp32 product) when embed_q is not null.
__global__ void k_embed(const uint16_t* __restrict__ embed, const int8_t* __restrict__ embed_q,
                        const float* __restrict__ embed_s, const int32_t* __restrict__ tok,
                        int vocab, int D, float* __restrict__ res, unsigned* status) {
  const int b = blockIdx.x;
  pdl_wait();
  pdl_release();
  int t = tok[b];
  if (t < 0 || t >= vocab) {
    if (threadIdx.x == 0) atomicOr(status, 2u);
    t = t < 0 ? 0 : vocab - 1;
  }
  if (embed_q) {
    const float sc = embed_s[t];
    for (int k = threadIdx.x; k < D; k += blockDim.x)
      res[size_t(b) * D + k] = sc * float(embed_q[size_t(t) * D + k]);
  } else {
    for (int k = threadIdx.x; k < D; k += blockDim.x)
      res[size_t(b) * D + k] = h2f(embed[size_t(t) * D + k]);
  }
}

// grid (rows), 256 threads.  Per-row int8 quantisation of an fp16 matrix: scale =
// max|row| / 127 (fp32 divide; 1 for an all-zero row), code = round-half-even(w /
// scale) clamped to [-127, 127], decided in fp32 (the activation quantiser's rule).
__global__ void __launch_bounds__(256) k_quant_rows(const uint16_t* __restrict__ w, int cols,
                                                    int8_t* __restrict__ q, float* __restrict__ scale) {
  __shared__ float red[32];
  const size_t r = blockIdx.x;
  float am = 0.f;
  for (int k = threadIdx.x; k < cols; k += blockDim.x) am = fmaxf(am, fabsf(h2f(w[r * cols + k])));
  am = block_max(am, red);
  const float sx = am > 0.f ? __fdiv_rn(am, 127.f) : 1.f;
  const float rcp = __frcp_rn(sx);
  for (int k = threadIdx.x; k < cols; k += blockDim.x)
    q[r * cols + k] = am > 0.f ? int8_t(quant_code_bits(h2f(w[r * cols + k]), sx, rcp)) : int8_t(0);
  if (threadIdx.x == 0) scale[r] = sx;
}

struct HeadArgs {
  int D, vocab, batch;
  const float* res;        // [B][D]
  const uint16_t* normf_w; // [D]
  const uint16_t* embed;   // [V][D] fp16, or
  const int8_t* embed_q;   // [V][D] int8 codes (when not null) with
  const float* embed_s;    // [V] fp32 row scales
  float* logits;           // [B][V] or null
  float* part_val;         // [B][gridDim.x]
  int* part_idx;           // [B][gridDim.x]
};

constexpr int kHeadWarps = 8;
constexpr int kHeadBatch = 8;   // batch rows per block (grid.y covers the rest)

DFSSM_DEV bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// grid (nblk, ceil(B/8)).  Each block recomputes the final RMSNorm of its batch rows
// (fp64, kept as fp32), streams its share of LM-head rows (one warp per row,
// 16-byte loads, fp32 accumulation) and keeps the best (logit, id) per batch row;
// the lowest id wins ties.
template <bool Q8>
__global__ void __launch_bounds__(kHeadWarps * 32) k_lmhead(HeadArgs a) {
  extern __shared__ __align__(16) float xf[];   // [8][D]
  __shared__ double red[32];
  __shared__ float wbest[kHeadWarps][kHeadBatch];
  __shared__ int wbesti[kHeadWarps][kHeadBatch];
  const int b0 = blockIdx.y * kHeadBatch;
  pdl_wait();
  pdl_release();
  const int nb = min(kHeadBatch, a.batch - b0);
  const int D = a.D;
  for (int bb = 0; bb < nb; ++bb) {
    const float* v = a.res + size_t(b0 + bb) * D;
    double ss = 0.0;
    for (int k = threadIdx.x; k < D; k += blockDim.x) ss = fma(double(v[k]), double(v[k]), ss);
    ss = block_sum_d(ss, red);
    const double rs = 1.0 / sqrt(ss / double(D) + kEpsD);
    for (int k = threadIdx.x; k < D; k += blockDim.x)
      xf[bb * D + k] = float((double(v[k]) * rs) * h2d(a.normf_w[k]));
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float best[kHeadBatch];
  int besti[kHeadBatch];
#pragma unroll
  for (int bb = 0; bb < kHeadBatch; ++bb) { best[bb] = -INFINITY; besti[bb] = 0x7fffffff; }
  const int nwarps = gridDim.x * kHeadWarps;
  for (int v = blockIdx.x * kHeadWarps + warp; v < a.vocab; v += nwarps) {
    float s[kHeadBatch];
#pragma unroll
    for (int bb = 0; bb < kHeadBatch; ++bb) s[bb] = 0.f;
    for (int c = lane; c < D / 8; c += 32) {
      float wf[8];
      if constexpr (Q8) {
        i8x8_to_float(__ldg(reinterpret_cast<const uint2*>(a.embed_q + size_t(v) * D) + c), wf);
      } else {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(a.embed + size_t(v) * D) + c);
        const __half2* wh = reinterpret_cast<const __half2*>(&w);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(wh[i]);
          wf[2 * i] = f.x;
          wf[2 * i + 1] = f.y;
        }
      }
#pragma unroll
      for (int bb = 0; bb < kHeadBatch; ++bb) {
        if (bb < nb) {
          const float4 x0 = reinterpret_cast<const float4*>(xf + bb * D + c * 8)[0];
          const float4 x1 = reinterpret_cast<const float4*>(xf + bb * D + c * 8)[1];
          float t = s[bb];
          t = fmaf(wf[0], x0.x, t); t = fmaf(wf[1], x0.y, t);
          t = fmaf(wf[2], x0.z, t); t = fmaf(wf[3], x0.w, t);
          t = fmaf(wf[4], x1.x, t); t = fmaf(wf[5], x1.y, t);
          t = fmaf(wf[6], x1.z, t); t = fmaf(wf[7], x1.w, t);
          s[bb] = t;
        }
      }
    }
#pragma unroll
    for (int bb = 0; bb < kHeadBatch; ++bb) {
      if (bb < nb) {
        const float l = Q8 ? warp_sum(s[bb]) * a.embed_s[v] : warp_sum(s[bb]);
        if (a.logits && lane == 0) a.logits[size_t(b0 + bb) * a.vocab + v] = l;
        if (better(l, v, best[bb], besti[bb])) { best[bb] = l; besti[bb] = v; }
      }
    }
  }
  if (lane == 0) {
    for (int bb = 0; bb < kHeadBatch; ++bb) { wbest[warp][bb] = best[bb]; wbesti[warp][bb] = besti[bb]; }
  }
  __syncthreads();
  if (threadIdx.x < nb) {
    const int bb = threadIdx.x;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int w = 0; w < kHeadWarps; ++w)
      if (better(wbest[w][bb], wbesti[w][bb], bv, bi)) { bv = wbest[w][bb]; bi = wbesti[w][bb]; }
    a.part_val[size_t(b0 + bb) * gridDim.x + blockIdx.x] = bv;
    a.part_idx[size_t(b0 + bb) * gridDim.x + blockIdx.x] = bi;
  }
}
// Tensor-core LM head for batches: grid (ceil(B / (8 NB)), gy).  Blocks with the same
// blockIdx.y read the same vocabulary rows and are launched next to each other, so
// the rows come from HBM about once.  A block normalises its 8 NB batch rows (fp64,
// kept as fp32, as k_lmhead) and splits each value into fp16 hi + lo parts
// (x = hi + lo to 2^-22 relative), so that the fp16 tensor-core products of the fp16
// head rows with both parts are exact and only the fp32 accumulation rounds.  Each
// warp owns 16-row vocabulary tiles (tile = 8 blockIdx.y + warp, + 8 gy, ...); per
// 64-column chunk, lane (g, t) loads 16 bytes x 2 of rows g and g + 8 at columns
// 16 t.. (coalesced, three chunks ahead) and runs four m16n8k16 MMAs per batch n-tile
// and part.  The MMA's k index i maps to column 64 c + 16 t + 4 s + (i & 1) + 2 (i >> 3)
// for A and B alike, so the chunk's 64 columns are each summed once.  Per batch row
// the block keeps the best (logit, id), lowest id on ties.
template <int NB, bool Q8>
__global__ void __launch_bounds__(kHeadWarps * 32) k_lmhead_tc(HeadArgs a) {
  extern __shared__ __align__(16) uint32_t xsw[];         // [2][8 NB][XS] words: hi rows, then lo rows
  __shared__ float wbest[kHeadWarps][8 * NB];
  __shared__ int wbesti[kHeadWarps][8 * NB];
  const int D = a.D, XS = D / 2 + 2;                       // row stride in words (== 2 mod 32)
  pdl_wait();
  pdl_release();
  const int b0 = blockIdx.x * 8 * NB;
  const int nb = min(8 * NB, a.batch - b0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  uint16_t* xh = reinterpret_cast<uint16_t*>(xsw);
  uint16_t* xl = reinterpret_cast<uint16_t*>(xsw + 8 * NB * XS);
  for (int rr = warp; rr < 8 * NB; rr += kHeadWarps) {
    if (rr < nb) {
      const float* v = a.res + size_t(b0 + rr) * D;
      double ss = 0.0;
      for (int k = lane; k < D; k += 32) ss = fma(double(v[k]), double(v[k]), ss);
      ss = warp_sum_d(ss);
      const double rs = 1.0 / sqrt(ss / double(D) + kEpsD);
      for (int k = lane; k < D; k += 32) {
        const float xv = float((double(v[k]) * rs) * h2d(a.normf_w[k]));
        const __half hi = __float2half_rn(xv);
        xh[rr * 2 * XS + k] = __half_as_ushort(hi);
        xl[rr * 2 * XS + k] = f2h(xv - __half2float(hi));
      }
    } else {
      for (int k = lane; k < D; k += 32) xh[rr * 2 * XS + k] = xl[rr * 2 * XS + k] = 0;
    }
  }
  __syncthreads();

  float best[NB][2];
  int besti[NB][2];
#pragma unroll
  for (int n = 0; n < NB; ++n) best[n][0] = best[n][1] = -INFINITY, besti[n][0] = besti[n][1] = 0x7fffffff;
  const int ntiles = (a.vocab + 15) / 16, nch = D / 64;
  const uint2* xh2 = reinterpret_cast<const uint2*>(xsw) + g * (XS / 2) + 4 * t;
  const uint2* xl2 = reinterpret_cast<const uint2*>(xsw + 8 * NB * XS) + g * (XS / 2) + 4 * t;
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  for (int tile = blockIdx.y * kHeadWarps + warp; tile < ntiles; tile += gridDim.y * kHeadWarps) {
    const int v0 = tile * 16 + g, v1 = v0 + 8;
    // fp16 rows: 2 x 16 bytes per 64-column chunk and lane; int8 rows: 16 bytes
    constexpr int kLV = Q8 ? 1 : 2;
    const uint4* r0 = Q8 ? reinterpret_cast<const uint4*>(a.embed_q + size_t(min(v0, a.vocab - 1)) * D) + t
                         : reinterpret_cast<const uint4*>(a.embed + size_t(min(v0, a.vocab - 1)) * D) + 2 * t;
    const uint4* r1 = Q8 ? reinterpret_cast<const uint4*>(a.embed_q + size_t(min(v1, a.vocab - 1)) * D) + t
                         : reinterpret_cast<const uint4*>(a.embed + size_t(min(v1, a.vocab - 1)) * D) + 2 * t;
    const bool ok0 = v0 < a.vocab, ok1 = v1 < a.vocab;
    // acc: one 64-column chunk's tensor-core sums; tot: the chunks' sum, taken with
    // round-to-nearest fp32 adds.  The tensor cores' own fp32 accumulation does not
    // round to nearest, and chained over a whole row (~256 MMAs at d_model 2048) it
    // biased logits toward zero by ~1.5e-5 relative; eight MMAs per chain keep that
    // bias near the fp32 rounding of the sum.
    float acc[NB][4], tot[NB][4];
#pragma unroll
    for (int n = 0; n < NB; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[n][e] = tot[n][e] = 0.f;
    // rows g and g + 8, 64-column chunks in a 4-slot register ring, three chunks ahead
    uint4 ring[4][2 * kLV];
    auto fetch = [&](uint4 (&dst)[2 * kLV], int c) {
#pragma unroll
      for (int i = 0; i < kLV; ++i) {
        dst[i] = ok0 ? __ldg(r0 + 4 * kLV * c + i) : z4;
        dst[kLV + i] = ok1 ? __ldg(r1 + 4 * kLV * c + i) : z4;
      }
    };
#pragma unroll
    for (int u = 0; u < 3; ++u)
      if (u < nch) fetch(ring[u], u);
    for (int c0 = 0; c0 < nch; c0 += 4) {      // nch is a multiple of 4 (D % 256 == 0)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u;
        if (c + 3 < nch) fetch(ring[(u + 3) & 3], c + 3);
        const uint4* cur = ring[u];
        uint32_t p0[8], p1[8];
        if constexpr (Q8) {   // 16 int8 columns per row -> 8 exact fp16 pairs
          const uint32_t w0[4] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w};
          const uint32_t w1[4] = {cur[1].x, cur[1].y, cur[1].z, cur[1].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            i8x4_to_half2x2(w0[i], p0[2 * i], p0[2 * i + 1]);
            i8x4_to_half2x2(w1[i], p1[2 * i], p1[2 * i + 1]);
          }
        } else {              // rows g and g + 8: two 16-byte vectors each
          const uint32_t q0[8] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w, cur[1].x, cur[1].y, cur[1].z, cur[1].w};
          const uint32_t q1[8] = {cur[2].x, cur[2].y, cur[2].z, cur[2].w, cur[3].x, cur[3].y, cur[3].z, cur[3].w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            p0[i] = q0[i];
            p1[i] = q1[i];
          }
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t af[4] = {p0[2 * s], p1[2 * s], p0[2 * s + 1], p1[2 * s + 1]};
#pragma unroll
          for (int n = 0; n < NB; ++n) {
            const uint2 bh = xh2[n * 8 * (XS / 2) + 16 * c + s];
            const uint2 bl = xl2[n * 8 * (XS / 2) + 16 * c + s];
            mma_f16_16816(acc[n], af, bh.x, bh.y);
            mma_f16_16816(acc[n], af, bl.x, bl.y);
          }
        }
#pragma unroll
        for (int n = 0; n < NB; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            tot[n][e] += acc[n][e];
            acc[n][e] = 0.f;
          }
      }
    }
#pragma unroll
    for (int n = 0; n < NB; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[n][e] = tot[n][e];
    if constexpr (Q8) {      // logit = row scale * (codes . x)
      const float s0 = ok0 ? a.embed_s[v0] : 0.f, s1 = ok1 ? a.embed_s[v1] : 0.f;
#pragma unroll
      for (int n = 0; n < NB; ++n) {
        acc[n][0] *= s0;
        acc[n][1] *= s0;
        acc[n][2] *= s1;
        acc[n][3] *= s1;
      }
    }
#pragma unroll
    for (int n = 0; n < NB; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int bc = n * 8 + 2 * t + e;
        if (bc < nb) {
          if (ok0) {
            if (a.logits) a.logits[size_t(b0 + bc) * a.vocab + v0] = acc[n][e];
            if (better(acc[n][e], v0, best[n][e], besti[n][e])) { best[n][e] = acc[n][e]; besti[n][e] = v0; }
          }
          if (ok1) {
            if (a.logits) a.logits[size_t(b0 + bc) * a.vocab + v1] = acc[n][2 + e];
            if (better(acc[n][2 + e], v1, best[n][e], besti[n][e])) { best[n][e] = acc[n][2 + e]; besti[n][e] = v1; }
          }
        }
      }
  }
  // best over the lanes of equal t (they hold the same batch columns), then over warps
#pragma unroll
  for (int n = 0; n < NB; ++n)
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best[n][e], o);
        const int oi = __shfl_xor_sync(0xffffffffu, besti[n][e], o);
        if (better(ov, oi, best[n][e], besti[n][e])) { best[n][e] = ov; besti[n][e] = oi; }
      }
  if (g == 0) {
#pragma unroll
    for (int n = 0; n < NB; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        wbest[warp][n * 8 + 2 * t + e] = best[n][e];
        wbesti[warp][n * 8 + 2 * t + e] = besti[n][e];
      }
  }
  __syncthreads();
  if (threadIdx.x < nb) {
    const int bc = threadIdx.x;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int w = 0; w < kHeadWarps; ++w)
      if (better(wbest[w][bc], wbesti[w][bc], bv, bi)) { bv = wbest[w][bc]; bi = wbesti[w][bc]; }
    a.part_val[size_t(b0 + bc) * gridDim.y + blockIdx.y] = bv;
    a.part_idx[size_t(b0 + bc) * gridDim.y + blockIdx.y] = bi;
  }
}

// grid (B).  Reduces the per-block (logit, id) pairs of one batch row.
__global__ void k_argmax(const float* __restrict__ part_val, const int* __restrict__ part_idx,
                         int nparts, int32_t* __restrict__ tok_out) {
  __shared__ float sv[256];
  __shared__ int si[256];
  const int b = blockIdx.x;
  pdl_wait();
  pdl_release();
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) {
    const float v = part_val[size_t(b) * nparts + i];
    const int id = part_idx[size_t(b) * nparts + i];
    if (better(v, id, bv, bi)) { bv = v; bi = id; }
  }
  sv[threadIdx.x] = bv;
  si[threadIdx.x] = bi;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s && better(sv[threadIdx.x + s], si[threadIdx.x + s], sv[threadIdx.x], si[threadIdx.x])) {
      sv[threadIdx.x] = sv[threadIdx.x + s];
      si[threadIdx.x] = si[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) tok_out[b] = si[0] == 0x7fffffff ? 0 : si[0];
}

}  // namespace dfssm
