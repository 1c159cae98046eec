// DF-SSM decode-step kernels ("Density Field State Space Models", Section 3.2 Eq. 3,
// Section 3.3, Section 4.1, Appendix B).  Layer path, one launch per stage:
//   k_prologue  RMSNorm -> fp16 activation -> int8 codes -> LoRA stage 1 (A_q . x_q)
//   k_proj      1-bit scaffold on int8 tensor cores (0/1 sign bytes x exact activation
//               digit planes, exact integer accumulation) + LoRA stage 2 (fp64)
//               + epilogue (store | residual add | conv1d shift-register step)
//   k_ssm       selective-SSM state update + D skip + gate y * silu(z)
//   k_lmhead    final RMSNorm + tied fp16 LM head + per-block argmax; k_argmax finishes it
#pragma once

#include "common.cuh"

namespace dfssm {

// ------------------------------------------------------------------ packing

DFSSM_DEV float load_dense(const void* w, int dtype, size_t i) {
  return dtype == 0 ? h2f(reinterpret_cast<const uint16_t*>(w)[i])
                    : reinterpret_cast<const float*>(w)[i];
}

// Inverse of the tiled layout: (tile word, bit) -> (row, col) inside the matrix.
// Bit s + 8i of a lane's word kt is byte i of A-fragment register q = s & 3 of
// 32-column chunk ch = s >> 2 (m16n8k32 .s8 fragment: rows g / g+8, columns
// 4t + i / 16 + 4t + i).
DFSSM_DEV void tiled_coord(size_t word, int bit, int kgroups, int* row, int* col) {
  const size_t tile = word / kTileWords;
  const int within = int(word % kTileWords);
  const int lane = within >> 2, kt = within & 3;
  const int rt = int(tile / kgroups), kg = int(tile % kgroups);
  const int i = bit >> 3, s = bit & 7;
  const int ch = s >> 2, q = s & 3;
  const int g = lane >> 2, t = lane & 3;
  *row = rt * kTileRows + g + 8 * (q & 1);
  *col = kg * kTileCols + kt * 64 + ch * 32 + 16 * (q >> 1) + 4 * t + i;
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
  const void* src;        // mode 0: [B][K] fp32 (residual) or fp64 (gated value) to normalise
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

constexpr int kPrologueThreads = 256;
constexpr int kPrologueRowsPerBlock = kPrologueThreads / 32;  // one LoRA row per warp

// grid (max(1, ceil(rank/8)), B).  Every block recomputes the activation of its
// batch row (same arithmetic, same result); block 0 also writes the activation,
// its int8 codes and its digit planes, and each warp computes one LoRA row.
//   mode 0: x = fp16(src * (1/sqrt(mean(src^2) + eps)) * w), all in fp64
//   mode 1: x = src16
//   sx = max|x| / 127, xq = clamp(rint(x / sx), -127, 127) (fp32 decision)
//   acc[j] = sum_k A[j,k] xq[k] (exact), u[j] = acc[j] * sA[j] * sx (fp64)
template <typename SrcT, int MODE>
__global__ void __launch_bounds__(kPrologueThreads) k_prologue(PrologueArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int K = a.K;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);            // [K]
  int8_t* qs = reinterpret_cast<int8_t*>(smem + 2 * K);        // [K]
  __shared__ double redd[32];
  __shared__ float red[32];
  __shared__ int redi[32];
  const int b = blockIdx.y, tid = threadIdx.x;
  const bool writer = blockIdx.x == 0;

  if (MODE == 0) {
    const SrcT* v = reinterpret_cast<const SrcT*>(a.src) + size_t(b) * K;
    double ss = 0.0;
    for (int k = tid; k < K; k += blockDim.x) {
      const double t = double(v[k]);
      ss = fma(t, t, ss);
    }
    ss = block_sum_d(ss, redd);
    const double rs = 1.0 / sqrt(ss / double(K) + kEpsD);
    const float rs32 = float(rs);
    for (int k = tid; k < K; k += blockDim.x) {
      uint16_t h;
      if constexpr (sizeof(SrcT) == 4) h = norm_fp16(float(v[k]), rs, rs32, half_to_float_bits(a.w[k]));
      else h = d2h((double(v[k]) * rs) * h2d(a.w[k]));
      xs[k] = h;
      if (writer && a.x) a.x[size_t(b) * K + k] = h;
    }
  } else {
    for (int k = tid; k < K; k += blockDim.x) xs[k] = a.src16[size_t(b) * K + k];
  }
  __syncthreads();
  float am = 0.f;
  for (int k = tid; k < K; k += blockDim.x) am = fmaxf(am, fabsf(h2f(xs[k])));
  am = block_max(am, red);
  const float sx = am > 0.f ? __fdiv_rn(am, 127.f) : 1.f;
  int dsum[kDigits];
#pragma unroll
  for (int d = 0; d < kDigits; ++d) dsum[d] = 0;
  const float rcp = __frcp_rn(sx);
  for (int k = tid; k < K; k += blockDim.x) {
    const int8_t q = am > 0.f ? int8_t(quant_code_bits(half_to_float_bits(xs[k]), sx, rcp)) : int8_t(0);
    qs[k] = q;
    if (writer) {
      a.xq[size_t(b) * K + k] = q;
      uint32_t lo, hi;
      digits_of(xs[k], &lo, &hi);
      const uint32_t w6[kDigits] = {lo, lo >> 8, lo >> 16, lo >> 24, hi, hi >> 8};
#pragma unroll
      for (int d = 0; d < kDigits; ++d) {
        const int8_t dg = int8_t(w6[d] & 0xffu);
        a.xd[(size_t(b) * kDigits + d) * K + k] = dg;
        dsum[d] += dg;
      }
    }
  }
  if (writer) {
#pragma unroll
    for (int d = 0; d < kDigits; ++d) {
      const int t = block_sum_i(dsum[d], redi);
      if (tid == 0) a.xdsum[b * kDigits + d] = t;
    }
    if (tid == 0) a.sx[b] = sx;
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x * kPrologueRowsPerBlock + warp;
  if (j < a.rank) {
    const int* Arow = reinterpret_cast<const int*>(a.A + size_t(j) * K);
    const int* q4 = reinterpret_cast<const int*>(qs);
    int acc = 0;
    for (int i = lane; i < K / 4; i += 32) acc = __dp4a(Arow[i], q4[i], acc);
    acc = warp_sum_i(acc);
    if (lane == 0) {
      a.acc[size_t(b) * a.rank + j] = acc;
      a.u[size_t(b) * a.rank + j] = (double(acc) * h2d(a.sA[j])) * double(sx);
    }
  }
}

// ------------------------------------------------------------------ projection

enum { EPI_STORE = 0, EPI_RESID = 1, EPI_INPROJ = 2 };

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
  double* zx;             // EPI_INPROJ: fp64 [batch][rows]
  // EPI_INPROJ conv step over rows [conv_lo, conv_lo + conv_dim)
  int conv_lo, conv_dim;
  const uint16_t* conv_w;  // [conv_dim][4]
  const uint16_t* conv_b;  // [conv_dim]
  float* conv_state;       // fp32 [batch][3][conv_dim]
  double* xc;              // fp64 [batch][conv_dim]
};

constexpr int kProjWarps = 8;
constexpr int kProjThreads = kProjWarps * 32;

__host__ __device__ constexpr int proj_cols(int bt) { return ((kDigits * bt + 7) / 8) * 8; }
__host__ __device__ __forceinline__ int proj_dstride(int K) { return K + 16; }  // bytes; spreads banks
__host__ __device__ __forceinline__ size_t proj_smem_bytes(int K, int rank, int bt) {
  return size_t(proj_cols(bt)) * proj_dstride(K)                 // digit planes
         + size_t(8) * bt * (rank > 0 ? rank : 1)                 // u (fp64)
         + size_t(4) * kProjWarps * 16 * proj_cols(bt)            // int32 partials
         + size_t(4) * bt * kDigits;                              // digit sums
}

// Scaffold value of one row from its per-plane 0/1 sums q[d] = sum_k bit * D_d[k]:
// sum_k s[k] x[k] = 2^-24 * sum_d 256^d (2 q[d] - T[d]), exact in int64.
DFSSM_DEV double scaffold_value(const int (&q)[kDigits], const int* T) {
  long long S = 0;
#pragma unroll
  for (int d = kDigits - 1; d >= 0; --d) S = S * 256 + (2LL * q[d] - T[d]);
  return double(S) * (1.0 / 16777216.0);
}

// grid (row-tile blocks, ceil(batch/BT)).  A block stages the digit planes of its
// BT batch rows once and then loops over 16-row tiles rt = blockIdx.x, +gridDim.x,
// ...; per tile the 8 warps split K in 256-column groups.  Each warp expands its lane's 16-byte vector of
// sign words into 0/1 int8 A fragments (one shift + one mask per register) and
// runs m16n8k32 int8 MMAs against the activation digit planes; int32 partials are
// summed in a fixed order in shared memory, recombined exactly, and the epilogue
// adds the LoRA stage 2 in fp64.
template <int EPI, int BT>
__global__ void __launch_bounds__(kProjThreads) k_proj(ProjArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int NC = proj_cols(BT), NT = NC / 8;
  const int K = a.K, DS = proj_dstride(K), rk = a.rank > 0 ? a.rank : 1;
  int8_t* dg = reinterpret_cast<int8_t*>(smem);                                   // [NC][DS]
  double* us = reinterpret_cast<double*>(smem + size_t(NC) * DS);                 // [BT][rank]
  int* part = reinterpret_cast<int*>(us + BT * rk);                               // [warps][16][NC]
  int* T = part + kProjWarps * 16 * NC;                                           // [BT][kDigits]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b0 = blockIdx.y * BT;
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
  for (int rt = blockIdx.x; rt < ntiles; rt += gridDim.x) {
  int acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0;
  const uint4* tiles = reinterpret_cast<const uint4*>(a.bits) + size_t(rt) * kgroups * 32;
  for (int kg = warp; kg < kgroups; kg += kProjWarps) {
    const uint4 wv = __ldg(tiles + kg * 32 + lane);
    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t af[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) af[q] = sign_bytes(words[kt], 4 * ch + q);
        const int k0 = kg * kTileCols + kt * 64 + ch * 32 + 4 * t;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const int8_t* dr = dg + size_t(n * 8 + g) * DS + k0;
          const uint32_t bf0 = *reinterpret_cast<const uint32_t*>(dr);
          const uint32_t bf1 = *reinterpret_cast<const uint32_t*>(dr + 16);
          mma_s8_16832(acc[n], af, bf0, bf1);
        }
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    int* p = part + size_t(warp) * 16 * NC;
    p[g * NC + n * 8 + 2 * t] = acc[n][0];
    p[g * NC + n * 8 + 2 * t + 1] = acc[n][1];
    p[(g + 8) * NC + n * 8 + 2 * t] = acc[n][2];
    p[(g + 8) * NC + n * 8 + 2 * t + 1] = acc[n][3];
  }
  __syncthreads();

  for (int i = tid; i < 16 * BT; i += blockDim.x) {
    const int r = i / BT, bb = i % BT;
    const int o = rt * kTileRows + r, b = b0 + bb;
    if (o >= a.rows || b >= a.batch) continue;
    int q[kDigits];
#pragma unroll
    for (int d = 0; d < kDigits; ++d) {
      int s = 0;
#pragma unroll
      for (int w = 0; w < kProjWarps; ++w) s += part[(w * 16 + r) * NC + bb * kDigits + d];
      q[d] = s;
    }
    double y = h2d(a.alpha[o]) * scaffold_value(q, T + bb * kDigits);
    if (a.rank > 0) {
      const int8_t* Br = a.B + size_t(o) * a.rank;
      const double* ur = us + bb * a.rank;
      double l = 0.0;
      for (int j = 0; j < a.rank; ++j) l = fma(double(Br[j]), ur[j], l);
      y = fma(h2d(a.sB[o]), l, y);
    }
    const size_t oi = size_t(b) * a.rows + o;
    if (EPI == EPI_RESID) {
      a.out[oi] = float(double(a.out[oi]) + y);
    } else if (EPI == EPI_STORE) {
      a.out[oi] = float(y);
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
  __syncthreads();   // the partials of this tile are consumed before the next tile's
  }
}

// ------------------------------------------------------------------ SSM step

struct SsmArgs {
  int H, P, N, E, conv_dim, in_rows;
  const double* zx;      // fp64 [B][in_rows]
  const double* xc;      // fp64 [B][conv_dim]
  const float* dt_bias;
  const float* A_log;
  const float* D;
  float* state;          // fp32 [B][H][P][N]
  float* g;              // fp32 [B][E]
};

constexpr int kSsmThreads = 256;

// grid (H, B): one block per head and batch row.  One warp per state row of N fp32
// values (float4 per lane, four rows of a warp in flight together), arithmetic in
// fp64, state stored back in fp32:
//   dt = softplus(dt_raw + dt_bias), dA = exp(-dt * exp(A_log)),
//   h' = dA h + (x dt) B,  y = C . h' + D x,  g = y * silu(z) (stored fp32).
__global__ void __launch_bounds__(kSsmThreads) k_ssm(SsmArgs a) {
  extern __shared__ __align__(16) double sbc[];   // [2N]: B then C
  const int h = blockIdx.x, b = blockIdx.y;
  const double* xcb = a.xc + size_t(b) * a.conv_dim;
  for (int i = threadIdx.x; i < 2 * a.N; i += blockDim.x) sbc[i] = xcb[a.E + i];
  const double* zr = a.zx + size_t(b) * a.in_rows;
  const double dt = softplus_d(zr[a.E + a.conv_dim + h] + double(a.dt_bias[h]));
  const double dA = exp(dt * -exp(double(a.A_log[h])));
  const double Dh = a.D[h];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kW = kSsmThreads / 32;
  // warp w takes rows w, w + kW, ...; four rows at a time so that their state loads
  // are in flight together
  for (int r0 = warp; r0 < a.P; r0 += 4 * kW) {
    double xdt[4], y[4] = {0.0, 0.0, 0.0, 0.0};
    float4* st[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int p = min(r0 + i * kW, a.P - 1), e = h * a.P + p;
      xdt[i] = xcb[e] * dt;
      st[i] = reinterpret_cast<float4*>(a.state + ((size_t(b) * a.H + h) * a.P + p) * a.N);
    }
    for (int n4 = lane; n4 < a.N / 4; n4 += 32) {
      float4 hv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) hv[i] = st[i][n4];
      const double* Bv = sbc + 4 * n4;
      const double* Cv = sbc + a.N + 4 * n4;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (r0 + i * kW >= a.P) continue;
        const double h0 = fma(dA, double(hv[i].x), xdt[i] * Bv[0]);
        const double h1 = fma(dA, double(hv[i].y), xdt[i] * Bv[1]);
        const double h2 = fma(dA, double(hv[i].z), xdt[i] * Bv[2]);
        const double h3 = fma(dA, double(hv[i].w), xdt[i] * Bv[3]);
        y[i] = fma(Cv[0], h0, y[i]);
        y[i] = fma(Cv[1], h1, y[i]);
        y[i] = fma(Cv[2], h2, y[i]);
        y[i] = fma(Cv[3], h3, y[i]);
        st[i][n4] = make_float4(float(h0), float(h1), float(h2), float(h3));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) y[i] += __shfl_xor_sync(0xffffffffu, y[i], o);
    if (lane < 4 && r0 + lane * kW < a.P) {
      const int e = h * a.P + r0 + lane * kW;
      double yy = lane == 0 ? y[0] : lane == 1 ? y[1] : lane == 2 ? y[2] : y[3];
      yy = fma(Dh, xcb[e], yy);
      a.g[size_t(b) * a.E + e] = float(yy * silu_d(zr[e]));
    }
  }
}

// ------------------------------------------------------------------ embedding / LM head

__global__ void k_embed(const uint16_t* __restrict__ embed, const int32_t* __restrict__ tok,
                        int vocab, int D, float* __restrict__ res, unsigned* status) {
  const int b = blockIdx.x;
  int t = tok[b];
  if (t < 0 || t >= vocab) {
    if (threadIdx.x == 0) atomicOr(status, 2u);
    t = t < 0 ? 0 : vocab - 1;
  }
  for (int k = threadIdx.x; k < D; k += blockDim.x)
    res[size_t(b) * D + k] = h2f(embed[size_t(t) * D + k]);
}

struct HeadArgs {
  int D, vocab, batch;
  const float* res;        // [B][D]
  const uint16_t* normf_w; // [D]
  const uint16_t* embed;   // [V][D]
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
__global__ void __launch_bounds__(kHeadWarps * 32) k_lmhead(HeadArgs a) {
  extern __shared__ __align__(16) float xf[];   // [8][D]
  __shared__ double red[32];
  __shared__ float wbest[kHeadWarps][kHeadBatch];
  __shared__ int wbesti[kHeadWarps][kHeadBatch];
  const int b0 = blockIdx.y * kHeadBatch;
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
    const uint4* row = reinterpret_cast<const uint4*>(a.embed + size_t(v) * D);
    float s[kHeadBatch];
#pragma unroll
    for (int bb = 0; bb < kHeadBatch; ++bb) s[bb] = 0.f;
    for (int c = lane; c < D / 8; c += 32) {
      const uint4 w = __ldg(row + c);
      const __half2* wh = reinterpret_cast<const __half2*>(&w);
      float wf[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(wh[i]);
        wf[2 * i] = f.x;
        wf[2 * i + 1] = f.y;
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
        const float l = warp_sum(s[bb]);
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
// grid (B).  Reduces the per-block (logit, id) pairs of one batch row.
__global__ void k_argmax(const float* __restrict__ part_val, const int* __restrict__ part_idx,
                         int nparts, int32_t* __restrict__ tok_out) {
  __shared__ float sv[256];
  __shared__ int si[256];
  const int b = blockIdx.x;
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
