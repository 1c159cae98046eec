// C ABI of libdfssm.so: host-side argument validation, workspace layout and the
// launch sequences of the DF-SSM decode step.  Declarations and semantics: dfssm.h.
#include <cudaTypedefs.h>

#include <algorithm>
#include <array>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "dfssm.h"
#include "kernels.cuh"
#include "persistent.cuh"

using namespace dfssm;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return DFSSM_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE(cond, code, ...) \
  do {                           \
    if (!(cond)) return fail(code, __VA_ARGS__); \
  } while (0)

#define REQUIRE_PTR(p) \
  do { \
    REQUIRE((p) != nullptr, DFSSM_ERR_INVALID_ARG, "%s is NULL", #p); \
    REQUIRE(aligned16(p), DFSSM_ERR_MISALIGNED, "%s is not 16-byte aligned", #p); \
  } while (0)

#define CHECK_LAUNCH(what) \
  do { \
    cudaError_t e_ = cudaGetLastError(); \
    if (e_ != cudaSuccess) return fail(DFSSM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e_)); \
  } while (0)

// Kernels of the multi-launch chain are launched with programmatic stream
// serialization: each may start while the kernel before it still runs, does its setup
// and reads only weights until pdl_wait() (common.cuh), so the launch and the setup
// overlap the previous kernel's tail.  DFSSM_PDL=0 at compile time turns it off.
#ifndef DFSSM_PDL
#define DFSSM_PDL 1
#endif
template <typename... KArgs, typename... Args>
cudaError_t launch_chain(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         unsigned cluster_z, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[2];
  unsigned n = 0;
  if (DFSSM_PDL) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_z > 0) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = 1;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = cluster_z;
    ++n;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
#define CHAIN_LAUNCH(what, ...) \
  do { \
    cudaError_t e_ = launch_chain(__VA_ARGS__); \
    if (e_ != cudaSuccess) return fail(DFSSM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e_)); \
  } while (0)

constexpr size_t kNone = ~size_t(0);
constexpr int kHeadBlocks = 592;  // 4 per SM on a 148-SM B200

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Bump {
  size_t off = 0;
  size_t take(size_t bytes) {
    off = align256(off);
    size_t at = off;
    off += bytes;
    return at;
  }
};

size_t tiled_words(int rows, int cols) {
  return size_t((rows + kTileRows - 1) / kTileRows) * kTileRows * (cols / 32);
}

int check_proj(const dfssm_proj* p, int rank, const char* name) {
  REQUIRE(p != nullptr, DFSSM_ERR_INVALID_ARG, "%s: projection is NULL", name);
  REQUIRE(p->rows > 0 && p->cols > 0, DFSSM_ERR_INVALID_ARG, "%s: rows/cols must be positive", name);
  REQUIRE(p->cols % kTileCols == 0, DFSSM_ERR_UNSUPPORTED_SHAPE, "%s: cols (%d) must be a multiple of 256", name, p->cols);
  REQUIRE(p->cols <= 8192, DFSSM_ERR_UNSUPPORTED_SHAPE, "%s: cols (%d) > 8192", name, p->cols);
  REQUIRE(rank >= 0 && rank <= 128 && rank % 4 == 0, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "%s: rank (%d) must be in [0, 128] and a multiple of 4", name, rank);
  REQUIRE(p->bits && aligned16(p->bits), p->bits ? DFSSM_ERR_MISALIGNED : DFSSM_ERR_INVALID_ARG,
          "%s: bits NULL or misaligned", name);
  REQUIRE(p->alpha && aligned16(p->alpha), p->alpha ? DFSSM_ERR_MISALIGNED : DFSSM_ERR_INVALID_ARG,
          "%s: alpha NULL or misaligned", name);
  if (rank > 0) {
    REQUIRE(p->A && p->sA && p->B && p->sB, DFSSM_ERR_INVALID_ARG, "%s: LoRA pointers NULL with rank %d", name, rank);
    REQUIRE(aligned16(p->A) && aligned16(p->sA) && aligned16(p->B) && aligned16(p->sB),
            DFSSM_ERR_MISALIGNED, "%s: LoRA pointer not 16-byte aligned", name);
  }
  return DFSSM_OK;
}

int check_dims(const dfssm_dims* d) {
  REQUIRE(d != nullptr, DFSSM_ERR_INVALID_ARG, "dims is NULL");
  REQUIRE(d->batch > 0 && d->d_model > 0 && d->d_inner > 0 && d->nheads > 0 && d->headdim > 0 &&
              d->d_state > 0, DFSSM_ERR_INVALID_ARG, "dims must be positive");
  REQUIRE(d->ngroups == 1, DFSSM_ERR_UNSUPPORTED_SHAPE, "ngroups (%d) must be 1", d->ngroups);
  REQUIRE(d->d_conv == kConvW, DFSSM_ERR_UNSUPPORTED_SHAPE, "d_conv (%d) must be 4", d->d_conv);
  REQUIRE(d->nheads * d->headdim == d->d_inner, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "d_inner (%d) != nheads*headdim (%d)", d->d_inner, d->nheads * d->headdim);
  REQUIRE(d->d_model % kTileCols == 0 && d->d_inner % kTileCols == 0, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "d_model and d_inner must be multiples of 256");
  REQUIRE(d->d_model <= 8192 && d->d_inner <= 8192, DFSSM_ERR_UNSUPPORTED_SHAPE, "d_model/d_inner > 8192");
  REQUIRE(d->headdim % 16 == 0 && d->headdim <= 128, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "headdim (%d) must be a multiple of 16 and <= 128", d->headdim);
  REQUIRE(d->ssm_state_dtype == 0 || d->ssm_state_dtype == 1, DFSSM_ERR_INVALID_ARG,
          "ssm_state_dtype (%d) must be 0 (fp32) or 1 (fp16)", d->ssm_state_dtype);
  REQUIRE(d->df_chunk_codec == 0 || d->df_chunk_codec == 1, DFSSM_ERR_INVALID_ARG,
          "df_chunk_codec (%d) must be 0 or 1", d->df_chunk_codec);
  REQUIRE(d->d_state % 4 == 0 && d->d_state <= 256, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "d_state (%d) must be a multiple of 4 and <= 256", d->d_state);
  REQUIRE(d->rank >= 0 && d->rank <= 128 && d->rank % 4 == 0, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "rank (%d) must be in [0,128], multiple of 4", d->rank);
  return DFSSM_OK;
}

int in_rows(const dfssm_dims* d) { return 2 * d->d_inner + 2 * d->ngroups * d->d_state + d->nheads; }
int conv_dim(const dfssm_dims* d) { return d->d_inner + 2 * d->ngroups * d->d_state; }

int check_layer(const dfssm_dims* d, const dfssm_layer_weights* w, const dfssm_layer_state* s, int li) {
  REQUIRE(w != nullptr && s != nullptr, DFSSM_ERR_INVALID_ARG, "layer %d: weights/state NULL", li);
  int rc;
  if ((rc = check_proj(&w->in, d->rank, "in_proj")) != 0) return rc;
  if ((rc = check_proj(&w->out, d->rank, "out_proj")) != 0) return rc;
  REQUIRE(w->in.rows == in_rows(d) && w->in.cols == d->d_model, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "layer %d: in_proj is %dx%d, dims need %dx%d (check d_state/nheads)", li, w->in.rows,
          w->in.cols, in_rows(d), d->d_model);
  REQUIRE(w->out.rows == d->d_model && w->out.cols == d->d_inner, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "layer %d: out_proj is %dx%d, dims need %dx%d", li, w->out.rows, w->out.cols, d->d_model,
          d->d_inner);
  const void* ptrs[] = {w->prenorm_w, w->conv_w, w->conv_b, w->dt_bias, w->A_log, w->D, w->gnorm_w,
                        s->conv_state, s->ssm_state};
  const char* names[] = {"prenorm_w", "conv_w", "conv_b", "dt_bias", "A_log", "D", "gnorm_w",
                         "conv_state", "ssm_state"};
  for (int i = 0; i < 9; ++i) {
    REQUIRE(ptrs[i] != nullptr, DFSSM_ERR_INVALID_ARG, "layer %d: %s is NULL", li, names[i]);
    REQUIRE(aligned16(ptrs[i]), DFSSM_ERR_MISALIGNED, "layer %d: %s not 16-byte aligned", li, names[i]);
  }
  return DFSSM_OK;
}

void layer_layout(const dfssm_dims* d, int n_layer, int vocab, dfssm_ws_layout* L) {
  const size_t B = d->batch, D = d->d_model, E = d->d_inner, r = d->rank ? d->rank : 1;
  Bump bp;
  L->status = bp.take(256);
  L->x_in = bp.take(2 * B * D);
  L->xq_in = bp.take(B * D);
  L->sx_in = bp.take(4 * B);
  L->acc_in = bp.take(4 * B * r);
  L->u_in = bp.take(8 * B * r);
  L->xd_in = bp.take(B * kDigits * D);
  L->xdsum_in = bp.take(4 * B * kDigits);
  L->zxbcdt = bp.take(8 * B * in_rows(d));
  L->xc = bp.take(8 * B * conv_dim(d));
  L->g = bp.take(4 * B * E);
  L->x_out = bp.take(2 * B * E);
  L->xq_out = bp.take(B * E);
  L->sx_out = bp.take(4 * B);
  L->acc_out = bp.take(4 * B * r);
  L->u_out = bp.take(8 * B * r);
  L->xd_out = bp.take(B * kDigits * E);
  L->xdsum_out = bp.take(4 * B * kDigits);
  // internal scratch: persistent-kernel / LM-head words
  if (n_layer > 0) {
    L->res = bp.take(4 * B * D);
    L->scratch = bp.take(persistent_scratch_bytes(d->batch, d->d_model, d->d_inner, in_rows(d), kHeadBlocks));
  } else {
    L->res = kNone;
    L->scratch = bp.take(persistent_scratch_bytes(d->batch, d->d_model, d->d_inner, in_rows(d), 0));
  }
  // the batch-1 token kernel's control words follow the LM-head partials in the scratch
  L->control = L->scratch + align256(size_t(8) * B * (n_layer > 0 ? kHeadBlocks : 1));
  L->total_bytes = align256(bp.off);
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<unsigned char*>(ws) + off); }

struct Act {       // one activation's preprocessing outputs
  uint16_t* x; int8_t* xq; float* sx; int* acc; double* u; int8_t* xd; int* xdsum;
};

struct Bufs {
  unsigned* status;
  Act in, out;
  double* zxbcdt; double* xc; float* g;
  float* res; unsigned char* scratch;
};

Bufs bind(void* ws, const dfssm_ws_layout& L, const dfssm_dims* d) {
  Bufs b;
  b.status = at<unsigned>(ws, L.status);
  b.in = Act{at<uint16_t>(ws, L.x_in), at<int8_t>(ws, L.xq_in), at<float>(ws, L.sx_in), at<int>(ws, L.acc_in),
             at<double>(ws, L.u_in), at<int8_t>(ws, L.xd_in), at<int>(ws, L.xdsum_in)};
  b.out = Act{at<uint16_t>(ws, L.x_out), at<int8_t>(ws, L.xq_out), at<float>(ws, L.sx_out),
              at<int>(ws, L.acc_out), at<double>(ws, L.u_out), at<int8_t>(ws, L.xd_out),
              at<int>(ws, L.xdsum_out)};
  b.zxbcdt = at<double>(ws, L.zxbcdt);
  b.xc = at<double>(ws, L.xc);
  b.g = at<float>(ws, L.g);
  b.res = L.res == kNone ? nullptr : at<float>(ws, L.res);
  b.scratch = at<unsigned char>(ws, L.scratch);
  return b;
}

// ---- launch helpers ---------------------------------------------------------

template <int MODE>
int launch_prologue(int K, int rank, int batch, const float* src, const uint16_t* src16, const uint16_t* w,
                    const Act& o, const dfssm_proj* p, cudaStream_t st) {
  PrologueArgs a{};
  a.K = K; a.rank = rank; a.src = src; a.src16 = src16; a.w = w;
  a.x = o.x; a.xq = o.xq; a.sx = o.sx; a.xd = o.xd; a.xdsum = o.xdsum;
  a.A = p->A; a.sA = p->sA; a.acc = o.acc; a.u = o.u;
  // the API limits (K a multiple of 256 and <= 8192, rank <= 128) are the kernels'
  REQUIRE(K % (16 * kPrologueCQ) == 0 && K <= kPrologueCQ * kPrologueClThreads * kPrologueClVals &&
              K <= 4 * kPrologueRowThreads * kPrologueRowGroups && rank <= kPrologueMaxRank,
          DFSSM_ERR_UNSUPPORTED_SHAPE, "prologue: K (%d) or rank (%d) out of range", K, rank);
  if (batch >= kPrologueRowMinBatch) {
    const int g = (K + 4 * kPrologueRowThreads - 1) / (4 * kPrologueRowThreads);
    switch (g) {
      case 1: CHAIN_LAUNCH("k_prologue_row", k_prologue_row<MODE, 1>, dim3(batch), dim3(kPrologueRowThreads), 0, st, 0, a); break;
      case 2: CHAIN_LAUNCH("k_prologue_row", k_prologue_row<MODE, 2>, dim3(batch), dim3(kPrologueRowThreads), 0, st, 0, a); break;
      case 3: CHAIN_LAUNCH("k_prologue_row", k_prologue_row<MODE, 3>, dim3(batch), dim3(kPrologueRowThreads), 0, st, 0, a); break;
      default: CHAIN_LAUNCH("k_prologue_row", k_prologue_row<MODE, 4>, dim3(batch), dim3(kPrologueRowThreads), 0, st, 0, a); break;
    }
    return DFSSM_OK;
  }
  const int v = (K / kPrologueCQ + kPrologueClThreads - 1) / kPrologueClThreads;
  switch (v) {
    case 1: CHAIN_LAUNCH("k_prologue_cl", k_prologue_cl<MODE, 1>, dim3(kPrologueCQ, batch), dim3(kPrologueClThreads), 0, st, 0, a); break;
    case 2: CHAIN_LAUNCH("k_prologue_cl", k_prologue_cl<MODE, 2>, dim3(kPrologueCQ, batch), dim3(kPrologueClThreads), 0, st, 0, a); break;
    case 3: CHAIN_LAUNCH("k_prologue_cl", k_prologue_cl<MODE, 3>, dim3(kPrologueCQ, batch), dim3(kPrologueClThreads), 0, st, 0, a); break;
    default: CHAIN_LAUNCH("k_prologue_cl", k_prologue_cl<MODE, 4>, dim3(kPrologueCQ, batch), dim3(kPrologueClThreads), 0, st, 0, a); break;
  }
  return DFSSM_OK;
}

constexpr size_t kProjSmemCap = 200 * 1024;

int pick_bt(int batch, int K, int rank) {
  // at most 4 batch rows per block: two blocks (32 warps) fit an SM, which hides
  // more latency than the better A-fragment reuse of 8 rows (measured)
  int bt = batch <= 1 ? 1 : batch <= 2 ? 2 : 4;
  while (bt > 1 && proj_smem_bytes(K, rank, bt) > kProjSmemCap) bt >>= 1;
  return bt;
}

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = 0;
  }
  return dev;
}

// SM count of the current device, cached per device.
int sm_count() {
  static std::mutex mu;
  static std::vector<std::array<int, 2>> cache;   // device, SMs
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& c : cache)
    if (c[0] == dev) return c[1];
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
    cudaGetLastError();
    v = 148;
  }
  cache.push_back({dev, v});
  return v;
}

// Resident blocks per SM of `kernel` with `threads` threads and `smem` bytes of
// dynamic shared memory on the current device, cached per (kernel, device, smem).
// The kernel's dynamic shared-memory limit is set to `smem` on every call (a cheap
// host call): the same kernel runs with several sizes, and a launch needs the
// limit at its own size.
int occupancy(const void* kernel, int threads, int smem) {
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    cudaGetLastError();
  struct Entry { const void* k; int dev, smem, blocks; };
  static std::mutex mu;
  static std::vector<Entry> cache;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& c : cache)
    if (c.k == kernel && c.dev == dev && c.smem == smem) return c.blocks;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, threads, size_t(smem)) != cudaSuccess || nb < 1) {
    cudaGetLastError();
    nb = 1;
  }
  cache.push_back({kernel, dev, smem, nb});
  return nb;
}

template <int EPI, int BT>
int launch_proj_bt(const ProjArgs& a, cudaStream_t st) {
  const size_t smem = proj_smem_bytes(a.K, a.rank, BT);
  // one wave of resident blocks; each reuses its staged digit planes over several tiles
  const int occ_blocks = occupancy(reinterpret_cast<const void*>(k_proj<EPI, BT>), kProjThreads, int(smem));
  const int ntiles = (a.rows + kTileRows - 1) / kTileRows, gy = (a.batch + BT - 1) / BT;
  const int wave = std::max(1, occ_blocks * sm_count() / gy);
  const int gx = std::max(1, std::min((ntiles + kProjWarps - 1) / kProjWarps, wave));
  dim3 grid(gx, gy);
  CHAIN_LAUNCH("k_proj", k_proj<EPI, BT>, grid, dim3(kProjThreads), smem, st, 0, a);
  return DFSSM_OK;
}

// Which scaffold kernel a batched projection takes: from batch 16 on the tcgen05
// tile kernel (k_proj_tc), below it the register-fragment mma.sync kernel (k_proj),
// whose per-row work suits a few batch rows.  DFSSM_PROJ_PATH=tc or =mma in the
// environment (read at every call) forces one of them, e.g. to compare the two.
int proj_path_override() {
  const char* e = getenv("DFSSM_PROJ_PATH");
  if (e && strcmp(e, "mma") == 0) return 1;
  if (e && strcmp(e, "tc") == 0) return 2;
  return 0;
}
constexpr int kTcMinBatch = 16;

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against
// the driver library), looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// The two TMA maps of k_proj_tc: the tiled sign words as [row tiles][K/256 x 128
// words] (box: 8 tiles x 128 words, no swizzle) and the digit planes as
// [batch x 6][K] bytes (box: N = 6 BG rows x 128 bytes, 128-byte swizzle).  Rows past
// the ends read as zeros.
int proj_tc_maps(const ProjArgs& a, int bg, CUtensorMap* bits, CUtensorMap* planes) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(DFSSM_ERR_CUDA, "k_proj_tc: cuTensorMapEncodeTiled is not available");
  REQUIRE(aligned16(a.bits) && aligned16(a.xd), DFSSM_ERR_MISALIGNED,
          "k_proj_tc: sign words and digit planes must be 16-byte aligned");
  const int kgroups = a.K / kTileCols, ntiles = (a.rows + kTileRows - 1) / kTileRows;
  const cuuint32_t estr[2] = {1, 1};
  const cuuint64_t bdim[2] = {cuuint64_t(kgroups) * kTileWords, cuuint64_t(ntiles)};
  const cuuint64_t bstride[1] = {cuuint64_t(kgroups) * kTileWords * 4};
  const cuuint32_t bbox[2] = {cuuint32_t(kTileWords), cuuint32_t(kTcTiles)};
  CUresult r = enc(bits, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(a.bits), bdim, bstride, bbox,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DFSSM_ERR_CUDA, "k_proj_tc: sign-word tensor map (%d)", int(r));
  const cuuint64_t pdim[2] = {cuuint64_t(a.K), cuuint64_t(a.batch) * kDigits};
  const cuuint64_t pstride[1] = {cuuint64_t(a.K)};
  const cuuint32_t pbox[2] = {128u, cuuint32_t(kDigits * bg)};
  r = enc(planes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(a.xd), pdim, pstride, pbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DFSSM_ERR_CUDA, "k_proj_tc: digit-plane tensor map (%d)", int(r));
  return DFSSM_OK;
}

// K split of a tcgen05 projection: double the CTAs sharing K (a cluster along z)
// while the grid still fits one wave of the SMs and every CTA keeps >= 2 k-blocks.
int proj_tc_split(int tiles, int kgroups) {
  int ks = 1;
  while (ks < kTcMaxSplit && tiles * ks * 2 <= sm_count() && kgroups % (ks * 2) == 0 && kgroups / (ks * 2) >= 2)
    ks *= 2;
  return ks;
}

template <int EPI, int BG>
int launch_proj_tc_bg(const ProjArgs& a, cudaStream_t st) {
  constexpr int smem = int(proj_tc_smem_bytes(BG));
  cudaError_t e = cudaFuncSetAttribute(k_proj_tc<EPI, BG>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return fail(DFSSM_ERR_CUDA, "k_proj_tc smem attribute: %s", cudaGetErrorString(e));
  REQUIRE(a.rank % 4 == 0, DFSSM_ERR_UNSUPPORTED_SHAPE, "k_proj_tc: rank %d", a.rank);
  CUtensorMap tb, tp;
  if (int rc = proj_tc_maps(a, BG, &tb, &tp)) return rc;
  const int mt = (a.rows + kTcM - 1) / kTcM, gb = (a.batch + BG - 1) / BG;
  const int ks = proj_tc_split(mt * gb, a.K / kTileCols);
  CHAIN_LAUNCH("k_proj_tc", k_proj_tc<EPI, BG>, dim3(mt, gb, ks), dim3(kTcThreads), size_t(smem), st, unsigned(ks),
               a, tb, tp);
  return DFSSM_OK;
}

template <int EPI>
int launch_proj(const ProjArgs& a, cudaStream_t st) {
  const int path = proj_path_override();
  if (path == 2 || (path == 0 && a.batch >= kTcMinBatch))
    return a.batch >= 32 ? launch_proj_tc_bg<EPI, 32>(a, st) : launch_proj_tc_bg<EPI, 16>(a, st);
  switch (pick_bt(a.batch, a.K, a.rank)) {
    case 1: return launch_proj_bt<EPI, 1>(a, st);
    case 2: return launch_proj_bt<EPI, 2>(a, st);
    default: return launch_proj_bt<EPI, 4>(a, st);
  }
}

ProjArgs proj_args(const dfssm_proj* p, int rank, int batch, const Act& act) {
  ProjArgs a{};
  a.rows = p->rows; a.K = p->cols; a.rank = rank; a.batch = batch;
  a.bits = p->bits; a.alpha = p->alpha; a.B = p->B; a.sB = p->sB;
  a.xd = act.xd; a.xdsum = act.xdsum; a.u = act.u;
  return a;
}

// LM head of the multi-launch path: the tensor-core kernel (16 or 8 batch rows per
// block) when its normalised rows fit in shared memory, else the fp32 kernel.
// `*nparts` receives the partials per batch row that k_argmax reduces.
constexpr size_t kHeadTcSmemCap = 200 * 1024;
size_t head_tc_smem(int D, int nb) { return size_t(2) * 8 * nb * (D + 4) * 2; }

template <int NB, bool Q8>
int launch_head_tc(const HeadArgs& h, cudaStream_t st, int* nparts) {
  const size_t smem = head_tc_smem(h.D, NB);
  const int occ_blocks = occupancy(reinterpret_cast<const void*>(k_lmhead_tc<NB, Q8>), kHeadWarps * 32, int(smem));
  const int gx = (h.batch + 8 * NB - 1) / (8 * NB);
  const int tiles = (h.vocab + 15) / 16;
  int gy = std::max(1, occ_blocks * sm_count() / gx);
  gy = std::min(gy, std::min(kHeadBlocks, (tiles + kHeadWarps - 1) / kHeadWarps));
  CHAIN_LAUNCH("k_lmhead_tc", k_lmhead_tc<NB, Q8>, dim3(gx, gy), dim3(kHeadWarps * 32), smem, st, 0, h);
  *nparts = gy;
  return DFSSM_OK;
}

template <bool Q8>
int launch_head_q(const HeadArgs& h, cudaStream_t st, int* nparts) {
  if (h.D % 256 == 0) {
    if (h.batch > 8 && head_tc_smem(h.D, 2) <= kHeadTcSmemCap) return launch_head_tc<2, Q8>(h, st, nparts);
    if (head_tc_smem(h.D, 1) <= kHeadTcSmemCap) return launch_head_tc<1, Q8>(h, st, nparts);
  }
  const size_t smem = size_t(4) * kHeadBatch * h.D;
  cudaFuncSetAttribute(k_lmhead<Q8>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  CHAIN_LAUNCH("k_lmhead", k_lmhead<Q8>, dim3(kHeadBlocks, (h.batch + kHeadBatch - 1) / kHeadBatch),
               dim3(kHeadWarps * 32), smem, st, 0, h);
  *nparts = kHeadBlocks;
  return DFSSM_OK;
}

int launch_head(const HeadArgs& h, cudaStream_t st, int* nparts) {
  return h.embed_q ? launch_head_q<true>(h, st, nparts) : launch_head_q<false>(h, st, nparts);
}

// SSM update of the multi-launch path: the streaming kernel when kSsmBufs buffers of
// an item's inputs fit and every bulk copy is 16-byte aligned, else k_ssm.
constexpr int kSsmStreamSmemCap = 96 * 1024;

template <int NCH, typename ST>
int launch_ssm_stream(const SsmArgs& sa, int smem, cudaStream_t st) {
  const int occ_blocks = occupancy(reinterpret_cast<const void*>(k_ssm_stream<NCH, ST>), kSsmStreamThreads, smem);
  const int items = sa.batch * sa.H * kSsmSplit;
  // every block's items fit its step-size table
  const int grid = std::max((items + kSsmStreamMaxItems - 1) / kSsmStreamMaxItems,
                            std::max(1, std::min(items, occ_blocks * sm_count())));
  CHAIN_LAUNCH("k_ssm_stream", k_ssm_stream<NCH, ST>, dim3(grid), dim3(kSsmStreamThreads), smem, st, 0, sa);
  return DFSSM_OK;
}

template <typename ST>
int launch_ssm_t(const SsmArgs& sa, cudaStream_t st) {
  const SsmItem it = ssm_item(sa.P, sa.N, int(sizeof(ST)));
  const int smem = kSsmBufs * ((it.bytes + 127) & ~127);
  const bool aligned = sa.P % kSsmSplit == 0 && it.rows % 2 == 0 &&
                       (size_t(sa.conv_dim) * 8) % 16 == 0 && (size_t(sa.in_rows) * 8) % 16 == 0 &&
                       (size_t(sa.E) * 8) % 16 == 0 && (size_t(sa.P) * 8) % 16 == 0 &&
                       (size_t(it.rows) * sa.N * sizeof(ST)) % 16 == 0 &&
                       aligned16(sa.state) && aligned16(sa.xc) && aligned16(sa.zx);
  if (aligned && smem <= kSsmStreamSmemCap) {
    if (sa.N <= 128) return launch_ssm_stream<1, ST>(sa, smem, st);
    return launch_ssm_stream<2, ST>(sa, smem, st);
  }
  if (sa.N <= 128) CHAIN_LAUNCH("k_ssm", k_ssm<1, ST>, dim3(sa.H, sa.batch), dim3(kSsmThreads), 0, st, 0, sa);
  else CHAIN_LAUNCH("k_ssm", k_ssm<2, ST>, dim3(sa.H, sa.batch), dim3(kSsmThreads), 0, st, 0, sa);
  return DFSSM_OK;
}

int launch_ssm(const SsmArgs& sa, cudaStream_t st) {
  return sa.state16 ? launch_ssm_t<__half>(sa, st) : launch_ssm_t<float>(sa, st);
}

// The layer as five dependent launches on one stream.
int layer_multikernel(const dfssm_dims* d, const dfssm_layer_weights* w, const dfssm_layer_state* s,
                      float* res, const Bufs& b, cudaStream_t st) {
  const int B = d->batch, D = d->d_model, E = d->d_inner, r = d->rank, C = conv_dim(d);
  int rc = launch_prologue<0>(D, r, B, res, nullptr, w->prenorm_w, b.in, &w->in, st);
  if (rc) return rc;
  ProjArgs pa = proj_args(&w->in, r, B, b.in);
  pa.status = b.status;
  pa.zx = b.zxbcdt;
  pa.conv_lo = E; pa.conv_dim = C; pa.conv_w = w->conv_w; pa.conv_b = w->conv_b;
  pa.conv_state = s->conv_state; pa.xc = b.xc;
  if ((rc = launch_proj<EPI_INPROJ>(pa, st))) return rc;
  SsmArgs sa{};
  sa.H = d->nheads; sa.P = d->headdim; sa.N = d->d_state; sa.E = E; sa.conv_dim = C; sa.in_rows = in_rows(d);
  sa.zx = b.zxbcdt; sa.xc = b.xc; sa.dt_bias = w->dt_bias; sa.A_log = w->A_log; sa.D = w->D;
  sa.state = s->ssm_state; sa.state16 = d->ssm_state_dtype == 1;
  sa.g = b.g; sa.dt_lo = E + C; sa.batch = B; sa.status = b.status;
  if ((rc = launch_ssm(sa, st))) return rc;
  if ((rc = launch_prologue<0>(E, r, B, b.g, nullptr, w->gnorm_w, b.out, &w->out, st))) return rc;
  ProjArgs po = proj_args(&w->out, r, B, b.out);
  po.status = b.status;
  po.out = res;
  return launch_proj<EPI_RESID>(po, st);
}

// ---- prompt pass (prefill) --------------------------------------------------------

// Workspace of a prompt pass: the decode layout for B*T token rows, then the
// last-token residual rows [B][D] fp32 (model prefill).  `base` is the token-row
// layout (its total marks where the extra region starts).
struct PrefillLayout {
  dfssm_dims rows;          // dims with batch = B * T
  dfssm_ws_layout base;     // layout of the B*T token rows
  size_t last;              // [B][D] fp32
  size_t total;
};

PrefillLayout prefill_layout(const dfssm_dims* d, int T, int n_layer, int vocab) {
  PrefillLayout P;
  P.rows = *d;
  P.rows.batch = d->batch * T;
  layer_layout(&P.rows, n_layer, vocab, &P.base);
  P.last = P.base.total_bytes;
  P.total = align256(P.last + size_t(4) * d->batch * d->d_model);
  return P;
}

int check_prefill(const dfssm_dims* d, int T) {
  REQUIRE(T >= 1, DFSSM_ERR_INVALID_ARG, "prompt length T (%d) must be >= 1", T);
  REQUIRE(size_t(d->batch) * T <= 65535, DFSSM_ERR_UNSUPPORTED_SHAPE, "batch * T (%lld) > 65535",
          (long long)d->batch * T);
  REQUIRE(ssd_smem_bytes(d->headdim, d->d_state) <= 200 * 1024, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "headdim * d_state (%d x %d) too large for the prompt-pass scan", d->headdim, d->d_state);
  REQUIRE(!d->df_chunk_codec || d->headdim <= kSsdThreads, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "the chunk-boundary codec takes headdim <= %d (%d)", kSsdThreads, d->headdim);
  return DFSSM_OK;
}

// One layer over the prompt: six launches on one stream.
int layer_prefill_launch(const dfssm_dims* d, int T, const dfssm_layer_weights* w, const dfssm_layer_state* s,
                         float* res, const Bufs& b, cudaStream_t st) {
  const int BT = d->batch * T, D = d->d_model, E = d->d_inner, r = d->rank, C = conv_dim(d);
  int rc = launch_prologue<0>(D, r, BT, res, nullptr, w->prenorm_w, b.in, &w->in, st);
  if (rc) return rc;
  ProjArgs pa = proj_args(&w->in, r, BT, b.in);
  pa.status = b.status;
  pa.zx = b.zxbcdt;
  if ((rc = launch_proj<EPI_ZX>(pa, st))) return rc;
  PrefillArgs fa{};
  fa.B = d->batch; fa.T = T; fa.H = d->nheads; fa.P = d->headdim; fa.N = d->d_state; fa.E = E; fa.C = C;
  fa.in_rows = in_rows(d); fa.zx = b.zxbcdt; fa.conv_w = w->conv_w; fa.conv_b = w->conv_b;
  fa.conv_state = s->conv_state; fa.xc = b.xc; fa.dt_bias = w->dt_bias; fa.A_log = w->A_log; fa.D = w->D;
  fa.state = s->ssm_state; fa.state16 = d->ssm_state_dtype == 1; fa.g = b.g; fa.df = d->df_chunk_codec != 0;
  k_conv_seq<<<dim3((C + 255) / 256, d->batch), 256, 0, st>>>(fa);
  CHECK_LAUNCH("k_conv_seq");
  const int smem = int(ssd_smem_bytes(fa.P, fa.N));
  if (fa.state16) {
    cudaFuncSetAttribute(k_ssd<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    k_ssd<__half><<<dim3(fa.H, d->batch), kSsdThreads, smem, st>>>(fa);
  } else {
    cudaFuncSetAttribute(k_ssd<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    k_ssd<float><<<dim3(fa.H, d->batch), kSsdThreads, smem, st>>>(fa);
  }
  CHECK_LAUNCH("k_ssd");
  if ((rc = launch_prologue<0>(E, r, BT, b.g, nullptr, w->gnorm_w, b.out, &w->out, st))) return rc;
  ProjArgs po = proj_args(&w->out, r, BT, b.out);
  po.status = b.status;
  po.out = res;
  return launch_proj<EPI_RESID>(po, st);
}

// ---- persistent whole-token kernel (batch 1) ------------------------------------


struct PPlan {
  bool ok = false;
  bool spec = false;   // the compile-time shape instantiation applies
  int grid = 0, Q = 0;
  PSmem sm{};
  char why[160] = {0};
};

int device_sm_count(int* dev, int* nsm, int* smem_optin) {
  cudaError_t e = cudaGetDevice(dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(nsm, cudaDevAttrMultiProcessorCount, *dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, *dev);
  return e == cudaSuccess ? 0 : -1;
}

// Clusters of Q persistent CTAs that can be resident at once (cached per device,
// cluster size and shared-memory size; the query is not a stream operation).
using PKernel = void (*)(PParams);
PKernel persistent_kernel(bool spec, bool q8 = false) {
  if (q8) return spec ? k_decode_persistent<Shape2048, true> : k_decode_persistent<ShapeAny, true>;
  return spec ? k_decode_persistent<Shape2048, false> : k_decode_persistent<ShapeAny, false>;
}

int max_active_clusters(int dev, int Q, int smem, bool spec) {
  static std::mutex mu;
  static std::vector<std::array<int, 5>> cache;   // dev, Q, smem, spec, result
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& c : cache)
    if (c[0] == dev && c[1] == Q && c[2] == smem && c[3] == int(spec)) return c[4];
  int n = 0;
  const PKernel kfn = persistent_kernel(spec);
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = unsigned(Q);
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(unsigned(Q));
    cfg.blockDim = dim3(kPBlock);
    cfg.dynamicSmemBytes = size_t(smem);
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(kfn), &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cache.push_back({dev, Q, smem, int(spec), n});
  return n;
}

bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// Whether (and how) one token of these dims runs as the persistent kernel.
PPlan plan_persistent(const dfssm_dims* d) {
  PPlan p;
  auto no = [&](const char* why) {
    snprintf(p.why, sizeof p.why, "%s", why);
    return p;
  };
  int dev = 0, nsm = 0, optin = 0;
  if (device_sm_count(&dev, &nsm, &optin)) return no("device query failed");
  const int D = d->d_model, E = d->d_inner, H = d->nheads, N = d->d_state, R = d->rank, P = d->headdim;
  if (d->batch != 1) return no("batch != 1");
  if (d->ssm_state_dtype != 0) return no("the token kernel holds fp32 SSM state");
  if (N % 16 || H % 16) return no("d_state and nheads must be multiples of 16");
  if (R != 0 && (!pow2(R) || R < 8 || R > kPThreads)) return no("rank must be 0 or a power of two in [8, 512]");
  if (D > kPMaxK || E > kPMaxK) return no("d_model and d_inner must be <= 4096");
  const int units = E / 16, out_tiles = D / 16, nbc = 2 * N / 16;
  // Clusters of 4 or 8 CTAs: the larger co-resident grid wins (clusters of 4 first on a
  // tie), so that every CTA gets as few SSM units and out_proj tiles as possible.
  int best_grid = 0, best_Q = 0, best_U = 0;
  // DFSSM_TOKEN_MAX_CTAS caps the grid (a diagnostic: a smaller co-resident grid can
  // be launched under a profiler); unset, the largest co-resident grid is used.
  int cap = kPlanSMs;
  if (const char* e = getenv("DFSSM_TOKEN_MAX_CTAS")) cap = std::max(4, std::min(kPlanSMs, atoi(e)));
  for (int Q : {4, 8}) {
    int U = 0;
    const int probe = std::min(kPlanSMs / Q, std::min(units, out_tiles) / Q) * Q;
    if (probe < Q) continue;
    for (int c = 0; c < probe; ++c) U = std::max(U, assign_cta(c, probe, Q, units, P, nbc, out_tiles).nu);
    const PSmem m = plan_smem(D, E, H, N, R, Q, U);
    if (m.total + int(sizeof(PParams)) + 1024 > optin || m.head_slots < 2) continue;
    const bool spec = D == Shape2048::D && E == Shape2048::E && H == Shape2048::H && P == Shape2048::P &&
                      N == Shape2048::N && R == Shape2048::R && Q == Shape2048::Q && U == Shape2048::U;
    const int maxc = max_active_clusters(dev, Q, m.total, spec);
    const int grid = std::min(std::min(maxc, cap / Q), std::min(units, out_tiles) / Q) * Q;
    if (grid > best_grid) {
      best_grid = grid;
      best_Q = Q;
      int U2 = 0;
      for (int c = 0; c < grid; ++c) U2 = std::max(U2, assign_cta(c, grid, Q, units, P, nbc, out_tiles).nu);
      best_U = U2;
    }
  }
  if (best_grid < 4) return no("no co-resident cluster of persistent CTAs");
  const int Q = best_Q, grid = best_grid;
  p.sm = plan_smem(D, E, H, N, R, Q, best_U);
  const PSmem& m = p.sm;
  p.spec = D == Shape2048::D && E == Shape2048::E && H == Shape2048::H && P == Shape2048::P && N == Shape2048::N &&
           R == Shape2048::R && Q == Shape2048::Q && best_U == Shape2048::U;
  if (p.spec && std::memcmp(&p.sm, &Shape2048::kPlan, sizeof(PSmem)) != 0) return no("compile-time plan mismatch");
  if (m.total + int(sizeof(PParams)) + 1024 > optin) return no("shared memory plan exceeds the per-block limit");
  if (m.head_slots < 2) return no("fewer than two LM-head chunk slots fit in shared memory");
  if (max_active_clusters(dev, Q, m.total, p.spec) * Q < grid) return no("the final plan does not stay co-resident");
  for (int c = 0; c < grid; ++c) {
    const PWork w = assign_cta(c, grid, Q, units, P, nbc, out_tiles);
    if (w.nu < 1 || w.nu > kPMaxUnits) return no("SSM row units per CTA out of range");
    if (w.no < 1 || w.no > kPMaxOutTiles) return no("out_proj tiles per CTA out of range");
    if (w.NS > kPMaxSharedTiles || w.ns > kPMaxShared || w.ntile > kPMaxInTiles) return no("too many in_proj tiles");
    if (w.h1 - w.h0 + 1 > kPMaxHeads) return no("too many heads per CTA");
  }
  p.grid = grid;
  p.Q = Q;
  p.ok = true;
  return p;
}

PLayer player(const dfssm_layer_weights& w, const dfssm_layer_state& s) {
  PLayer L;
  L.prenorm_w = w.prenorm_w;
  L.in_bits = w.in.bits; L.in_alpha = w.in.alpha; L.in_A = w.in.A; L.in_sA = w.in.sA; L.in_B = w.in.B;
  L.in_sB = w.in.sB;
  L.conv_w = w.conv_w; L.conv_b = w.conv_b; L.dt_bias = w.dt_bias; L.A_log = w.A_log; L.D = w.D;
  L.gnorm_w = w.gnorm_w;
  L.out_bits = w.out.bits; L.out_alpha = w.out.alpha; L.out_A = w.out.A; L.out_sA = w.out.sA;
  L.out_B = w.out.B; L.out_sB = w.out.sB;
  L.conv_state = s.conv_state; L.ssm_state = static_cast<float*>(s.ssm_state);   // fp32 (planner)
  return L;
}

// Launch one token (model mode) or one layer step (layer mode) as the persistent kernel.
// The tied embedding / LM-head matrix: fp16 rows, or int8 codes with fp32 row scales.
struct EmbedRef {
  const uint16_t* f16 = nullptr;
  const int8_t* q = nullptr;
  const float* s = nullptr;
};

#ifdef DFSSM_PHASE_TIMERS
// Phase-timer build: per-CTA cycle sums of the token kernel in a file-scope device
// array (the address is looked up per device and cached).
static __device__ unsigned long long g_phase_cycles[kPlanSMs * kPhaseSlots];
std::mutex g_phase_mu;
void* g_phase_addr[64] = {};

int phase_buffer(unsigned long long** out) {
  const int dev = current_device();
  REQUIRE(dev >= 0 && dev < 64, DFSSM_ERR_DEVICE, "device %d beyond the 64 supported", dev);
  std::lock_guard<std::mutex> lock(g_phase_mu);
  if (g_phase_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_phase_cycles);
    if (e != cudaSuccess || p == nullptr) return fail(DFSSM_ERR_CUDA, "phase timers: %s", cudaGetErrorString(e));
    g_phase_addr[dev] = p;
  }
  *out = static_cast<unsigned long long*>(g_phase_addr[dev]);
  return DFSSM_OK;
}
#endif

int launch_persistent(const PPlan& plan, const dfssm_dims* d, int n_layer, int vocab,
                      const dfssm_layer_weights* layers, const dfssm_layer_state* states, const EmbedRef& emb,
                      const uint16_t* normf_w, const int32_t* tok_in, int32_t* tok_out, float* logits,
                      float* residual, void* ws, const dfssm_ws_layout& WL, int head_blocks, cudaStream_t st) {
  static_assert(sizeof(PParams) < 32000, "kernel parameter block too large");
  PParams a;
  std::memset(&a, 0, sizeof a);
  const int D = d->d_model, E = d->d_inner, N = d->d_state, R = d->rank;
  a.n_layer = n_layer; a.D = D; a.E = E; a.H = d->nheads; a.P = d->headdim; a.N = N; a.R = R;
  a.in_rows = in_rows(d); a.C = conv_dim(d); a.vocab = vocab;
  a.kg_in = D / kTileCols; a.kg_out = E / kTileCols;
  a.units = E / 16; a.grid = plan.grid; a.Q = plan.Q;
  a.n_bc_tiles = 2 * N / 16; a.dt_tile0 = (2 * E + 2 * N) / 16; a.out_tiles = D / 16;
  a.SD = D / plan.Q; a.SE = E / plan.Q;
  a.layer_mode = residual != nullptr;
  a.sm = plan.sm;
  a.embed = emb.f16; a.embed_q = emb.q; a.embed_s = emb.s;
  a.normf_w = normf_w; a.tok_in = tok_in; a.tok_out = tok_out; a.logits = logits;
  a.residual = residual;
  (void)head_blocks;
  unsigned char* pbase = at<unsigned char>(ws, WL.control);
  a.status = at<unsigned>(ws, WL.status);
  a.ctl = reinterpret_cast<unsigned*>(pbase);
  unsigned long long* wd = reinterpret_cast<unsigned long long*>(pbase + 256);
  a.x_r = wd;      wd += D;
  a.x_rs = wd;     wd += 2 * plan.grid;
  a.x_g = wd;      wd += E;
  a.x_gs = wd;     wd += 2 * plan.grid;
  a.x_head = wd;   wd += 2 * plan.grid;
  Bufs b = bind(ws, WL, d);
  a.d_x_in = b.in.x; a.d_xq_in = b.in.xq; a.d_sx_in = b.in.sx; a.d_acc_in = b.in.acc; a.d_u_in = b.in.u;
  a.d_xd_in = b.in.xd; a.d_xdsum_in = b.in.xdsum; a.d_zx = b.zxbcdt; a.d_xc = b.xc; a.d_g = b.g;
  a.d_x_out = b.out.x; a.d_xq_out = b.out.xq; a.d_sx_out = b.out.sx; a.d_acc_out = b.out.acc;
  a.d_u_out = b.out.u; a.d_xd_out = b.out.xd; a.d_xdsum_out = b.out.xdsum; a.d_res = b.res;
  for (int l = 0; l < n_layer; ++l) a.L[l] = player(layers[l], states[l]);
#ifdef DFSSM_PHASE_TIMERS
  {
    int rc = phase_buffer(&a.phase);
    if (rc) return rc;
  }
#endif
  const PKernel kfn = persistent_kernel(plan.spec, emb.q != nullptr);
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, plan.sm.total);
  if (e != cudaSuccess) return fail(DFSSM_ERR_CUDA, "persistent smem attribute: %s", cudaGetErrorString(e));
  // clusters of Q CTAs, all co-resident (cooperative): the CTAs wait on one another
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = unsigned(plan.Q);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeCooperative;
  at[1].val.cooperative = 1;
  cfg.gridDim = dim3(unsigned(plan.grid));
  cfg.blockDim = dim3(kPBlock);
  cfg.dynamicSmemBytes = size_t(plan.sm.total);
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kfn, a);
  if (e != cudaSuccess) return fail(DFSSM_ERR_CUDA, "persistent launch: %s", cudaGetErrorString(e));
  CHECK_LAUNCH("k_decode_persistent");
  return DFSSM_OK;
}

}  // namespace

extern "C" {

int dfssm_version(void) { return 210; }

int dfssm_phase_timers(uint64_t* out, int max_entries, int reset) {
#ifdef DFSSM_PHASE_TIMERS
  REQUIRE(max_entries >= 0, DFSSM_ERR_INVALID_ARG, "max_entries must be >= 0");
  unsigned long long* dev = nullptr;
  int rc = phase_buffer(&dev);
  if (rc) return rc;
  const int n = std::min(max_entries, kPlanSMs * kPhaseSlots);
  if (n > 0) {
    REQUIRE(out != nullptr, DFSSM_ERR_INVALID_ARG, "out is NULL");
    const cudaError_t e = cudaMemcpy(out, dev, sizeof(uint64_t) * n, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(DFSSM_ERR_CUDA, "phase timers: %s", cudaGetErrorString(e));
  }
  if (reset) {
    const cudaError_t e = cudaMemset(dev, 0, sizeof(uint64_t) * kPlanSMs * kPhaseSlots);
    if (e != cudaSuccess) return fail(DFSSM_ERR_CUDA, "phase timers: %s", cudaGetErrorString(e));
  }
  ok();
  return n;
#else
  (void)out; (void)max_entries; (void)reset;
  return fail(DFSSM_ERR_NOT_BUILT, "this library was built without DFSSM_PHASE_TIMERS");
#endif
}

int dfssm_model_decode_launches(const dfssm_dims* d, int n_layer, int vocab) {
  if (check_dims(d) || n_layer < 1 || n_layer > kMaxLayers || vocab < 1) return 0;
  if (plan_persistent(d).ok) return 1;
  return 1 + 5 * n_layer + 2;
}

const char* dfssm_last_error(void) { return g_last_error.c_str(); }

size_t dfssm_packed_words(int rows, int cols, int layout) {
  if (rows <= 0 || cols <= 0) return 0;
  if (layout == DFSSM_LAYOUT_ROWMAJOR) return cols % 32 ? 0 : size_t(rows) * (cols / 32);
  if (layout == DFSSM_LAYOUT_TILED) return cols % kTileCols ? 0 : tiled_words(rows, cols);
  return 0;
}

int dfssm_pack_weights(const void* w, int dtype, int rows, int cols, int layout, uint32_t* bits,
                       void* stream) {
  REQUIRE(rows > 0 && cols > 0, DFSSM_ERR_INVALID_ARG, "rows/cols must be positive");
  REQUIRE(dtype == DFSSM_DTYPE_F16 || dtype == DFSSM_DTYPE_F32, DFSSM_ERR_INVALID_ARG, "bad dtype %d", dtype);
  REQUIRE(layout == DFSSM_LAYOUT_ROWMAJOR || layout == DFSSM_LAYOUT_TILED, DFSSM_ERR_INVALID_ARG,
          "bad layout %d", layout);
  REQUIRE(cols % (layout == DFSSM_LAYOUT_TILED ? kTileCols : 32) == 0, DFSSM_ERR_UNSUPPORTED_SHAPE,
          "cols (%d) must be a multiple of %d", cols, layout == DFSSM_LAYOUT_TILED ? kTileCols : 32);
  REQUIRE_PTR(w);
  REQUIRE_PTR(bits);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = dfssm_packed_words(rows, cols, layout);
  const int blocks = int(std::min<size_t>((n + 255) / 256, 148 * 16));
  if (layout == DFSSM_LAYOUT_ROWMAJOR)
    k_pack_rowmajor<<<blocks, 256, 0, st>>>(w, dtype, rows, cols, bits);
  else
    k_pack_tiled<<<blocks, 256, 0, st>>>(w, dtype, rows, cols, bits, n);
  CHECK_LAUNCH("pack");
  return ok();
}

int dfssm_repack_bits(const uint32_t* rowmajor, int rows, int cols, uint32_t* tiled, void* stream) {
  REQUIRE(rows > 0 && cols > 0, DFSSM_ERR_INVALID_ARG, "rows/cols must be positive");
  REQUIRE(cols % kTileCols == 0, DFSSM_ERR_UNSUPPORTED_SHAPE, "cols (%d) must be a multiple of 256", cols);
  REQUIRE_PTR(rowmajor);
  REQUIRE_PTR(tiled);
  const size_t n = tiled_words(rows, cols);
  const int blocks = int(std::min<size_t>((n + 255) / 256, 148 * 16));
  k_repack_tiled<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(rowmajor, rows, cols, tiled, n);
  CHECK_LAUNCH("repack");
  return ok();
}

int dfssm_proj_workspace_layout(int rows, int cols, int rank, int batch, dfssm_ws_layout* L) {
  REQUIRE(L != nullptr, DFSSM_ERR_INVALID_ARG, "layout is NULL");
  REQUIRE(rows > 0 && cols > 0 && batch > 0 && rank >= 0, DFSSM_ERR_INVALID_ARG, "bad sizes");
  std::memset(L, 0xff, sizeof *L);
  const size_t B = batch, r = rank ? rank : 1;
  Bump bp;
  L->status = bp.take(256);
  L->xq_in = bp.take(B * cols);
  L->sx_in = bp.take(4 * B);
  L->acc_in = bp.take(4 * B * r);
  L->u_in = bp.take(8 * B * r);
  L->xd_in = bp.take(B * kDigits * cols);
  L->xdsum_in = bp.take(4 * B * kDigits);
  L->total_bytes = align256(bp.off);
  return ok();
}

size_t dfssm_proj_workspace_bytes(int rows, int cols, int rank, int batch) {
  dfssm_ws_layout L;
  if (dfssm_proj_workspace_layout(rows, cols, rank, batch, &L)) return 0;
  return L.total_bytes;
}

int dfssm_proj_forward(const dfssm_proj* p, int rank, int batch, const uint16_t* x, float* y, void* ws,
                       size_t ws_bytes, void* stream) {
  int rc = check_proj(p, rank, "proj");
  if (rc) return rc;
  REQUIRE(batch > 0, DFSSM_ERR_INVALID_ARG, "batch must be positive");
  REQUIRE_PTR(x);
  REQUIRE_PTR(y);
  REQUIRE_PTR(ws);
  dfssm_ws_layout L;
  dfssm_proj_workspace_layout(p->rows, p->cols, rank, batch, &L);
  REQUIRE(ws_bytes >= L.total_bytes, DFSSM_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", ws_bytes,
          L.total_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Act act{nullptr, at<int8_t>(ws, L.xq_in), at<float>(ws, L.sx_in), at<int>(ws, L.acc_in),
          at<double>(ws, L.u_in), at<int8_t>(ws, L.xd_in), at<int>(ws, L.xdsum_in)};
  if ((rc = launch_prologue<1>(p->cols, rank, batch, nullptr, x, nullptr, act, p, st))) return rc;
  ProjArgs a = proj_args(p, rank, batch, act);
  a.status = at<unsigned>(ws, L.status);
  a.out = y;
  if ((rc = launch_proj<EPI_STORE>(a, st))) return rc;
  return ok();
}

int dfssm_workspace_layout(const dfssm_dims* d, int n_layer, int vocab, dfssm_ws_layout* L) {
  int rc = check_dims(d);
  if (rc) return rc;
  REQUIRE(L != nullptr, DFSSM_ERR_INVALID_ARG, "layout is NULL");
  REQUIRE(n_layer >= 0 && vocab >= 0 && (n_layer == 0) == (vocab == 0), DFSSM_ERR_INVALID_ARG,
          "n_layer and vocab must both be 0 (layer step) or both positive (model decode)");
  layer_layout(d, n_layer, vocab, L);
  return ok();
}

size_t dfssm_workspace_bytes(const dfssm_dims* d, int n_layer, int vocab) {
  dfssm_ws_layout L;
  if (dfssm_workspace_layout(d, n_layer, vocab, &L)) return 0;
  return L.total_bytes;
}

int dfssm_layer_step(const dfssm_dims* d, const dfssm_layer_weights* w, const dfssm_layer_state* s,
                     float* residual, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_dims(d);
  if (rc) return rc;
  if ((rc = check_layer(d, w, s, 0))) return rc;
  REQUIRE_PTR(residual);
  REQUIRE_PTR(ws);
  dfssm_ws_layout L;
  layer_layout(d, 0, 0, &L);
  REQUIRE(ws_bytes >= L.total_bytes, DFSSM_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", ws_bytes,
          L.total_bytes);
  Bufs b = bind(ws, L, d);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const PPlan plan = plan_persistent(d);
  if (plan.ok) {
    if ((rc = launch_persistent(plan, d, 1, 0, w, s, EmbedRef{}, nullptr, nullptr, nullptr, nullptr, residual, ws, L,
                                0, st)))
      return rc;
  } else if ((rc = layer_multikernel(d, w, s, residual, b, st))) {
    return rc;
  }
  return ok();
}

}  // extern "C"

namespace {

int model_decode(const dfssm_dims* d, int n_layer, int vocab, const EmbedRef& emb,
                 const dfssm_layer_weights* layers, const dfssm_layer_state* states, const uint16_t* normf_w,
                 const int32_t* tok_in, int32_t* tok_out, float* logits, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_dims(d);
  if (rc) return rc;
  REQUIRE(n_layer >= 1 && n_layer <= kMaxLayers, DFSSM_ERR_INVALID_ARG, "n_layer (%d) must be in [1, %d]",
          n_layer, kMaxLayers);
  REQUIRE(vocab >= 1, DFSSM_ERR_INVALID_ARG, "vocab must be positive");
  REQUIRE(layers != nullptr && states != nullptr, DFSSM_ERR_INVALID_ARG, "layers/states NULL");
  for (int l = 0; l < n_layer; ++l)
    if ((rc = check_layer(d, &layers[l], &states[l], l))) return rc;
  if (emb.q) {
    REQUIRE_PTR(emb.q);
    REQUIRE_PTR(emb.s);
  } else {
    REQUIRE_PTR(emb.f16);
  }
  REQUIRE_PTR(normf_w);
  REQUIRE_PTR(tok_in);
  REQUIRE_PTR(tok_out);
  REQUIRE(logits == nullptr || aligned16(logits), DFSSM_ERR_MISALIGNED, "logits not 16-byte aligned");
  REQUIRE_PTR(ws);
  dfssm_ws_layout L;
  layer_layout(d, n_layer, vocab, &L);
  REQUIRE(ws_bytes >= L.total_bytes, DFSSM_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", ws_bytes,
          L.total_bytes);
  Bufs b = bind(ws, L, d);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int B = d->batch, D = d->d_model;
  const PPlan plan = plan_persistent(d);
  if (plan.ok) {
    if ((rc = launch_persistent(plan, d, n_layer, vocab, layers, states, emb, normf_w, tok_in, tok_out, logits,
                                nullptr, ws, L, kHeadBlocks, st)))
      return rc;
    return ok();
  }
  CHAIN_LAUNCH("k_embed", k_embed, dim3(B), dim3(256), 0, st, 0, emb.f16, emb.q, emb.s, tok_in, vocab, D, b.res,
               b.status);
  for (int l = 0; l < n_layer; ++l)
    if ((rc = layer_multikernel(d, &layers[l], &states[l], b.res, b, st))) return rc;
  float* part_val = reinterpret_cast<float*>(b.scratch);
  int* part_idx = reinterpret_cast<int*>(b.scratch + size_t(4) * B * kHeadBlocks);
  HeadArgs h{};
  h.D = D; h.vocab = vocab; h.batch = B; h.res = b.res; h.normf_w = normf_w;
  h.embed = emb.f16; h.embed_q = emb.q; h.embed_s = emb.s;
  h.logits = logits; h.part_val = part_val; h.part_idx = part_idx;
  int nparts = kHeadBlocks;
  if ((rc = launch_head(h, st, &nparts))) return rc;
  CHAIN_LAUNCH("k_argmax", k_argmax, dim3(B), dim3(256), 0, st, 0, part_val, part_idx, nparts, tok_out);
  return ok();
}

}  // namespace

extern "C" {

int dfssm_model_decode(const dfssm_dims* d, int n_layer, int vocab, const uint16_t* embed,
                       const dfssm_layer_weights* layers, const dfssm_layer_state* states,
                       const uint16_t* normf_w, const int32_t* tok_in, int32_t* tok_out, float* logits,
                       void* ws, size_t ws_bytes, void* stream) {
  EmbedRef e;
  e.f16 = embed;
  REQUIRE_PTR(embed);
  return model_decode(d, n_layer, vocab, e, layers, states, normf_w, tok_in, tok_out, logits, ws, ws_bytes,
                      stream);
}

int dfssm_model_decode_q8(const dfssm_dims* d, int n_layer, int vocab, const int8_t* embed_q,
                          const float* embed_scale, const dfssm_layer_weights* layers,
                          const dfssm_layer_state* states, const uint16_t* normf_w, const int32_t* tok_in,
                          int32_t* tok_out, float* logits, void* ws, size_t ws_bytes, void* stream) {
  REQUIRE_PTR(embed_q);
  REQUIRE_PTR(embed_scale);
  EmbedRef e;
  e.q = embed_q;
  e.s = embed_scale;
  return model_decode(d, n_layer, vocab, e, layers, states, normf_w, tok_in, tok_out, logits, ws, ws_bytes,
                      stream);
}

int dfssm_quantize_rows_int8(const uint16_t* w, int rows, int cols, int8_t* q, float* scale, void* stream) {
  REQUIRE(rows > 0 && cols > 0, DFSSM_ERR_INVALID_ARG, "rows/cols must be positive");
  REQUIRE_PTR(w);
  REQUIRE_PTR(q);
  REQUIRE_PTR(scale);
  k_quant_rows<<<rows, 256, 0, static_cast<cudaStream_t>(stream)>>>(w, cols, q, scale);
  CHECK_LAUNCH("k_quant_rows");
  return ok();
}

}  // extern "C"

// ---- projection with library-owned scratch ----------------------------------
//
// For callers that cannot call cudaMalloc: dfssm_proj_forward needs a workspace,
// and some callers have no way to obtain one (a plugin whose host framework hands
// it no allocator, or a latency-critical thread that must not risk the device-wide
// synchronisation cudaMalloc/cudaFree can cause).  This variant runs the same
// kernels with its scratch in a fixed file-scope device array instead.

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB per device, held until exit
constexpr int kNoAllocMaxDevices = 64;

// The name below is only a host-side handle; its device address is looked up once
// per device with cudaGetSymbolAddress and cached.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};

int noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DFSSM_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  REQUIRE(dev >= 0 && dev < kNoAllocMaxDevices, DFSSM_ERR_DEVICE, "device %d beyond the %d supported", dev,
          kNoAllocMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(DFSSM_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return DFSSM_OK;
}

}  // namespace

extern "C" int dfssm_proj_forward_noalloc(const dfssm_proj* p, int rank, int batch, const uint16_t* x,
                                          float* y, void* stream) {
  int rc = check_proj(p, rank, "proj");
  if (rc) return rc;
  REQUIRE(batch > 0, DFSSM_ERR_INVALID_ARG, "batch must be positive");
  REQUIRE_PTR(x);
  REQUIRE_PTR(y);
  dfssm_ws_layout L;
  if ((rc = dfssm_proj_workspace_layout(p->rows, p->cols, rank, batch, &L))) return rc;
  REQUIRE(L.total_bytes <= kNoAllocScratchBytes, DFSSM_ERR_WORKSPACE_TOO_SMALL,
          "this projection needs %zu bytes of scratch but the built-in scratch holds %zu bytes; "
          "use dfssm_proj_forward with a caller workspace", L.total_bytes, kNoAllocScratchBytes);
  void* ws = nullptr;
  if ((rc = noalloc_scratch(&ws))) return rc;
  // Every region of the projection's scratch is written before it is read, so
  // nothing left by an earlier call needs clearing.
  return dfssm_proj_forward(p, rank, batch, x, y, ws, kNoAllocScratchBytes, stream);
}

// ---- prompt pass (prefill) ----------------------------------------------------------

extern "C" {

int dfssm_prefill_workspace_layout(const dfssm_dims* d, int T, int n_layer, int vocab, dfssm_ws_layout* out) {
  int rc = check_dims(d);
  if (rc) return rc;
  if ((rc = check_prefill(d, T))) return rc;
  REQUIRE(out != nullptr, DFSSM_ERR_INVALID_ARG, "layout is NULL");
  REQUIRE(n_layer >= 0 && vocab >= 0 && (n_layer == 0) == (vocab == 0), DFSSM_ERR_INVALID_ARG,
          "n_layer and vocab must both be 0 (layer prefill) or both positive (model prefill)");
  const PrefillLayout P = prefill_layout(d, T, n_layer, vocab);
  *out = P.base;
  out->total_bytes = P.total;
  return ok();
}

size_t dfssm_prefill_workspace_bytes(const dfssm_dims* d, int T, int n_layer, int vocab) {
  dfssm_ws_layout L;
  if (dfssm_prefill_workspace_layout(d, T, n_layer, vocab, &L)) return 0;
  return L.total_bytes;
}

int dfssm_layer_prefill(const dfssm_dims* d, int T, const dfssm_layer_weights* w, const dfssm_layer_state* s,
                        float* residual, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_dims(d);
  if (rc) return rc;
  if ((rc = check_prefill(d, T))) return rc;
  if ((rc = check_layer(d, w, s, 0))) return rc;
  REQUIRE_PTR(residual);
  REQUIRE_PTR(ws);
  const PrefillLayout P = prefill_layout(d, T, 0, 0);
  REQUIRE(ws_bytes >= P.total, DFSSM_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", ws_bytes, P.total);
  const Bufs b = bind(ws, P.base, &P.rows);
  if ((rc = layer_prefill_launch(d, T, w, s, residual, b, static_cast<cudaStream_t>(stream)))) return rc;
  return ok();
}

int dfssm_model_prefill(const dfssm_dims* d, int n_layer, int vocab, const uint16_t* embed,
                        const dfssm_layer_weights* layers, const dfssm_layer_state* states, const uint16_t* normf_w,
                        int T, const int32_t* tokens, int32_t* tok_out, float* logits, void* ws, size_t ws_bytes,
                        void* stream) {
  int rc = check_dims(d);
  if (rc) return rc;
  if ((rc = check_prefill(d, T))) return rc;
  REQUIRE(n_layer >= 1 && n_layer <= kMaxLayers, DFSSM_ERR_INVALID_ARG, "n_layer (%d) must be in [1, %d]",
          n_layer, kMaxLayers);
  REQUIRE(vocab >= 1, DFSSM_ERR_INVALID_ARG, "vocab must be positive");
  REQUIRE(layers != nullptr && states != nullptr, DFSSM_ERR_INVALID_ARG, "layers/states NULL");
  for (int l = 0; l < n_layer; ++l)
    if ((rc = check_layer(d, &layers[l], &states[l], l))) return rc;
  REQUIRE_PTR(embed);
  REQUIRE_PTR(normf_w);
  REQUIRE_PTR(tokens);
  REQUIRE_PTR(tok_out);
  REQUIRE(logits == nullptr || aligned16(logits), DFSSM_ERR_MISALIGNED, "logits not 16-byte aligned");
  REQUIRE_PTR(ws);
  const PrefillLayout P = prefill_layout(d, T, n_layer, vocab);
  REQUIRE(ws_bytes >= P.total, DFSSM_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", ws_bytes, P.total);
  const Bufs b = bind(ws, P.base, &P.rows);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int B = d->batch, D = d->d_model;
  k_embed<<<B * T, 256, 0, st>>>(embed, nullptr, nullptr, tokens, vocab, D, b.res, b.status);
  CHECK_LAUNCH("k_embed");
  for (int l = 0; l < n_layer; ++l)
    if ((rc = layer_prefill_launch(d, T, &layers[l], &states[l], b.res, b, st))) return rc;
  float* last = at<float>(ws, P.last);
  k_last_rows<<<B, 256, 0, st>>>(b.res, T, D, last);
  CHECK_LAUNCH("k_last_rows");
  float* part_val = reinterpret_cast<float*>(b.scratch);
  int* part_idx = reinterpret_cast<int*>(b.scratch + size_t(4) * B * kHeadBlocks);
  HeadArgs h{};
  h.D = D; h.vocab = vocab; h.batch = B; h.res = last; h.normf_w = normf_w;
  h.embed = embed; h.logits = logits; h.part_val = part_val; h.part_idx = part_idx;
  int nparts = kHeadBlocks;
  if ((rc = launch_head(h, st, &nparts))) return rc;
  CHAIN_LAUNCH("k_argmax", k_argmax, dim3(B), dim3(256), 0, st, 0, part_val, part_idx, nparts, tok_out);
  return ok();
}


// ---- density-field state codec -------------------------------------------------

int dfssm_df_field_words(int d_state) {
  REQUIRE(d_state >= 1, DFSSM_ERR_INVALID_ARG, "d_state (%d) must be >= 1", d_state);
  return df_field_words(d_state);
}

int dfssm_df_encode(const float* rows, int n_rows, int d_state, uint32_t* cells, float* lo, float* span,
                    float* rows_out, void* stream) {
  REQUIRE(rows && cells && lo && span && n_rows >= 0 && d_state >= 1, DFSSM_ERR_INVALID_ARG,
          "df_encode: null pointer or bad size (rows %d, d_state %d)", n_rows, d_state);
  if (n_rows == 0) return ok();
  k_df_encode<<<(n_rows + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(rows, n_rows, d_state, cells,
                                                                                      lo, span, rows_out);
  CHECK_LAUNCH("k_df_encode");
  return ok();
}

int dfssm_df_decode(const uint32_t* cells, const float* lo, const float* span, int n_rows, int d_state,
                    float* rows, void* stream) {
  REQUIRE(rows && cells && lo && span && n_rows >= 0 && d_state >= 1, DFSSM_ERR_INVALID_ARG,
          "df_decode: null pointer or bad size (rows %d, d_state %d)", n_rows, d_state);
  if (n_rows == 0) return ok();
  k_df_decode<<<(n_rows + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(cells, lo, span, n_rows,
                                                                                      d_state, rows);
  CHECK_LAUNCH("k_df_decode");
  return ok();
}

}  // extern "C"
