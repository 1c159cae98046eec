// Latency of the two exchange primitives the batch-1 token kernel is built from,
// measured on the device in isolation (no other work between rounds):
//   grid   : an all-gather of tagged 64-bit words over a cooperative grid -- each CTA
//            publishes its share of W words plus 2 partial words per round, every CTA
//            gathers all of them (each thread keeping all its loads in flight);
//   cluster: an all-to-all inside a cluster of 8 by st.async into every CTA's shared
//            memory, completion counted in bytes on the receiver's mbarrier.
// Every wait is bounded; the status word records a wait that gave up.  Rounds are
// timed with CUDA events over 2000 rounds.
#include <cstdio>
#include <cstdlib>
#include <cuda_runtime.h>

#define CK(x)                                                                          \
  do {                                                                                 \
    cudaError_t e_ = (x);                                                              \
    if (e_ != cudaSuccess) {                                                           \
      printf("CUDA %s at line %d\n", cudaGetErrorString(e_), __LINE__);                \
      exit(1);                                                                         \
    }                                                                                  \
  } while (0)

constexpr long long kSpin = 1LL << 20;

__device__ __forceinline__ void tw_put(unsigned long long* p, unsigned v, unsigned tag) {
  const unsigned long long w = ((unsigned long long)tag << 32) | v;
  asm volatile("st.volatile.global.u64 [%0], %1;" :: "l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ unsigned long long tw_load(const unsigned long long* p) {
  unsigned long long w;
  asm volatile("ld.volatile.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}

template <int MAXW>
__global__ void __launch_bounds__(512, 1) k_grid(unsigned long long* tw, int W, int iters, unsigned* status,
                                                 unsigned* sink) {
  const int G = gridDim.x, c = blockIdx.x, tid = threadIdx.x, T = blockDim.x;
  const int total = W + 2 * G;
  __shared__ unsigned sdat[4096 + 512];
  __shared__ int s_bad;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  unsigned acc = 0;
  const int w0 = int((long long)c * W / G), w1 = int((long long)(c + 1) * W / G);
  for (int i = 1; i <= iters; ++i) {
    unsigned long long* sl = tw + size_t(i & 1) * total;
    for (int k = w0 + tid; k < w1; k += T) tw_put(sl + k, k * 7u + i, i);
    if (tid < 2) tw_put(sl + W + 2 * c + tid, c + i, i);
    for (int base = 0; base < total; base += MAXW * T) {
      unsigned pend = 0;
#pragma unroll
      for (int j = 0; j < MAXW; ++j)
        if (base + tid + j * T < total) pend |= 1u << j;
      long long s = 0;
      while (pend) {
        unsigned long long w[MAXW];
#pragma unroll
        for (int j = 0; j < MAXW; ++j)
          if (pend & (1u << j)) w[j] = tw_load(sl + base + tid + j * T);
#pragma unroll
        for (int j = 0; j < MAXW; ++j)
          if ((pend & (1u << j)) && unsigned(w[j] >> 32) == unsigned(i)) {
            sdat[base + tid + j * T] = unsigned(w[j]);
            pend &= ~(1u << j);
          }
        if (pend && ++s > kSpin) {
          atomicOr(status, 1u);
          s_bad = 1;
          break;
        }
      }
    }
    __syncthreads();
    acc += sdat[(tid * 37) % total];
    if (s_bad) break;
  }
  if (acc == 0xdeadbeefu) sink[0] = acc;
}

__device__ __forceinline__ unsigned smem_u32(const void* p) { return unsigned(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ unsigned mapa(unsigned a, unsigned r) {
  unsigned o;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(o) : "r"(a), "r"(r));
  return o;
}
__device__ __forceinline__ bool try_wait_cl(unsigned bar, unsigned par) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(bar), "r"(par) : "memory");
  return ok != 0;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(512, 1) k_cluster(int words, int iters, unsigned* status, unsigned* sink) {
  __shared__ __align__(16) unsigned rx[2][8 * 256];
  __shared__ __align__(8) unsigned long long bar[2];
  __shared__ int s_bad;
  unsigned Q, r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(Q));
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_bad = 0;
    for (int b = 0; b < 2; ++b) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(smem_u32(&bar[b])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  cluster_sync();
  unsigned acc = 0;
  for (int i = 0; i < iters; ++i) {
    const int b = i & 1;
    const unsigned par = unsigned(i >> 1) & 1u;
    if (tid == 0)
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(&bar[b])),
                   "r"(unsigned(Q * words * 4)) : "memory");
    for (int k = tid; k < int(Q) * words; k += blockDim.x) {
      const unsigned dst = k / words, v = k % words;
      asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
                   :: "r"(mapa(smem_u32(&rx[b][r * words + v]), dst)), "r"(i + v), "r"(mapa(smem_u32(&bar[b]), dst))
                   : "memory");
    }
    if (tid == 0) {
      long long s = 0;
      while (!try_wait_cl(smem_u32(&bar[b]), par))
        if (++s > kSpin) {
          atomicOr(status, 2u);
          s_bad = 1;
          break;
        }
    }
    __syncthreads();
    acc += rx[b][(tid * 13) % (Q * words)];
    if (s_bad) break;
  }
  if (acc == 0xdeadbeefu) sink[0] = acc;
  cluster_sync();   // no CTA leaves while a peer may still write into it
}

int main() {
  CK(cudaSetDevice(0));
  unsigned long long* tw;
  unsigned *status, *sink;
  CK(cudaMalloc(&tw, size_t(2) * (4096 + 512) * 8));
  CK(cudaMalloc(&status, 4));
  CK(cudaMalloc(&sink, 4));
  const int iters = 2000;
  cudaEvent_t e0, e1;
  CK(cudaEventCreate(&e0));
  CK(cudaEventCreate(&e1));
  for (int G : {120, 128})
    for (int W : {2048, 4096}) {
      CK(cudaMemset(tw, 0, size_t(2) * (4096 + 512) * 8));
      CK(cudaMemset(status, 0, 4));
      void* args[] = {&tw, &W, (void*)&iters, &status, &sink};
      CK(cudaEventRecord(e0));
      CK(cudaLaunchCooperativeKernel((void*)k_grid<10>, G, 512, args, 0, 0));
      CK(cudaEventRecord(e1));
      CK(cudaEventSynchronize(e1));
      float ms;
      CK(cudaEventElapsedTime(&ms, e0, e1));
      unsigned st;
      CK(cudaMemcpy(&st, status, 4, cudaMemcpyDeviceToHost));
      printf("grid all-gather: %d CTAs x 512 threads, %d words + %d partial words per round: %.3f us/round (status %u)\n",
             G, W, 2 * G, ms * 1e3 / iters, st);
    }
  for (int words : {32, 256}) {
    CK(cudaMemset(status, 0, 4));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 8;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(120);
    cfg.blockDim = dim3(512);
    cfg.attrs = at;
    cfg.numAttrs = 1;
    CK(cudaEventRecord(e0));
    CK(cudaLaunchKernelEx(&cfg, k_cluster, words, iters, status, sink));
    CK(cudaEventRecord(e1));
    CK(cudaEventSynchronize(e1));
    float ms;
    CK(cudaEventElapsedTime(&ms, e0, e1));
    unsigned st;
    CK(cudaMemcpy(&st, status, 4, cudaMemcpyDeviceToHost));
    printf("cluster all-to-all (st.async, 8 CTAs x 512 threads): %d words per pair: %.3f us/round (status %u)\n", words,
           ms * 1e3 / iters, st);
  }
  return 0;
}
