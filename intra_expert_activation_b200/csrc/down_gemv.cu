// Down projection on CUDA cores for expert token groups with few tokens
// (decode): stream only the W_down rows in the group's active-neuron union
// with 128-bit loads and multiply them by the tokens' h values.
//
// This is the low-batch side of the pages' batch-size switch [gist.science
// EN "Uncovering Intra-expert Activation Sparsity for Efficient
// Mixture-of-Expert Model Execution", Technical Summary > Methodology >
// System Implementation in vLLM > "Dynamic Switching"]: with one to a few
// tokens per expert the down projection is a matrix-vector product whose
// cost is the bytes of the rows it reads ["Fused Up-Down Projection": only
// the active neurons' weights are fetched].
//
// Work unit: (group, slice of d_model columns), handled by one thread-block
// cluster of kCluster CTAs that split the union rows evenly; each warp walks
// its rows with an 8-deep unrolled stream of 16-byte loads (one 512-byte row
// segment per warp load), keeps fp32 partial sums in registers, the CTA sums
// its warps through shared memory, and rank 0 sums the CTAs of the cluster
// through distributed shared memory in rank order (deterministic) and writes
// Y[slot][columns]. Clusters walk units with a static stride.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCluster = 8;
constexpr int kUnroll = 8;
constexpr int kRowChunk = 2048;  // union positions staged in shared memory at a time

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <typename TW>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(b[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
};

// h of MT consecutive slots of one neuron row of H^T; entries past mt are 0.
template <typename TW, int MT>
__device__ __forceinline__ void load_h(const TW* p, int mt, float (&h)[MT]) {
  if constexpr (sizeof(TW) == 2) {
    static_assert(MT == 4 || MT == 8, "bf16 h vector");
    if constexpr (MT == 4) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
      const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
      const float2 a = __bfloat1622float2(b[0]), c = __bfloat1622float2(b[1]);
      h[0] = a.x; h[1] = a.y; h[2] = c.x; h[3] = c.y;
    } else {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
      float f[8];
      Vec<__nv_bfloat16>::unpack(u, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) h[i] = f[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < MT; i += 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(p + i));
      h[i] = v.x; h[i + 1] = v.y; h[i + 2] = v.z; h[i + 3] = v.w;
    }
  }
#pragma unroll
  for (int i = 0; i < MT; ++i)
    if (i >= mt) h[i] = 0.f;
}

template <typename TW, int MT>
__global__ void __launch_bounds__(kThreads)
    down_gemv_kernel(Dims dm, Workspace ws, const TW* __restrict__ Wd,
                     const TW* __restrict__ Wds) {
  constexpr int VEC = Vec<TW>::N;
  constexpr int SW = 32 * VEC;  // columns per slice: one 512-byte row segment
  __shared__ float red[kWarps][MT][SW];
  __shared__ float part[MT][SW];
  __shared__ int srows[kRowChunk];

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int cid = blockIdx.x / kCluster;
  const int ncl = gridDim.x / kCluster;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = dm.d;
  const int n_slices = d / SW;
  const int n_units = __ldcg(ws.meta + kMetaGemvCount) * n_slices;
  const size_t ld = static_cast<size_t>(dm.slots_total);
  const TW* ht = static_cast<const TW*>(ws.ht);

  for (int u = cid; u < n_units; u += ncl) {
    const int g = __ldcg(ws.gemv_list + u / n_slices);
    const int c0 = (u % n_slices) * SW;
    const Group gr = ws.groups[g];
    const bool shared = gr.expert >= dm.E;
    const int F_e = shared ? dm.Fs : dm.F;
    const TW* W = shared ? Wds + static_cast<size_t>(gr.expert - dm.E) * F_e * d
                         : Wd + static_cast<size_t>(gr.expert) * F_e * d;
    W += c0 + lane * VEC;
    const int cnt = __ldcg(ws.union_cnt + g);
    const int* rows = ws.union_rows + static_cast<size_t>(g) * dm.F_max;
    const int lo = static_cast<int>(static_cast<long long>(rank) * cnt / kCluster);
    const int hi = static_cast<int>(static_cast<long long>(rank + 1) * cnt / kCluster);

    for (int tp = 0; tp < gr.m; tp += MT) {
      const int mt = min(MT, gr.m - tp);
      const TW* hcol = ht + gr.slot0 + tp;
      float acc[MT][VEC];
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[t][v] = 0.f;

      for (int base = lo; base < hi; base += kRowChunk) {
        const int n = min(kRowChunk, hi - base);
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += kThreads) srows[i] = __ldcg(rows + base + i);
        __syncthreads();
        int i = warp;
        for (; i + kWarps * (kUnroll - 1) < n; i += kWarps * kUnroll) {
          uint4 wv[kUnroll];
          float hv[kUnroll][MT];
#pragma unroll
          for (int r = 0; r < kUnroll; ++r) {
            const int j = srows[i + kWarps * r];
            wv[r] = ld_stream(W + static_cast<size_t>(j) * d);
            load_h<TW, MT>(hcol + static_cast<size_t>(j) * ld, mt, hv[r]);
          }
#pragma unroll
          for (int r = 0; r < kUnroll; ++r) {
            float w[VEC];
            Vec<TW>::unpack(wv[r], w);
#pragma unroll
            for (int t = 0; t < MT; ++t)
#pragma unroll
              for (int v = 0; v < VEC; ++v) acc[t][v] = fmaf(hv[r][t], w[v], acc[t][v]);
          }
        }
        for (; i < n; i += kWarps) {
          const int j = srows[i];
          const uint4 wv = ld_stream(W + static_cast<size_t>(j) * d);
          float hv[MT];
          load_h<TW, MT>(hcol + static_cast<size_t>(j) * ld, mt, hv);
          float w[VEC];
          Vec<TW>::unpack(wv, w);
#pragma unroll
          for (int t = 0; t < MT; ++t)
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[t][v] = fmaf(hv[t], w[v], acc[t][v]);
        }
      }

      // CTA: sum the warps (fixed order)
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int v = 0; v < VEC; ++v) red[warp][t][lane * VEC + v] = acc[t][v];
      __syncthreads();
      for (int e = threadIdx.x; e < MT * SW; e += kThreads) {
        const int t = e / SW, c = e % SW;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w][t][c];
        part[t][c] = s;
      }
      // cluster: rank 0 sums the CTAs in rank order
      cluster.sync();
      if (rank == 0) {
        float* y = ws.y + static_cast<size_t>(gr.slot0 + tp) * d + c0;
        for (int e = threadIdx.x; e < mt * SW; e += kThreads) {
          const int t = e / SW, c = e % SW;
          float s = 0.f;
#pragma unroll
          for (int r = 0; r < kCluster; ++r) s += cluster.map_shared_rank(&part[0][0], r)[t * SW + c];
          y[static_cast<size_t>(t) * d + c] = s;
        }
      }
      cluster.sync();
    }
  }
}

}  // namespace

cudaError_t launch_down_gemv(const Dims& dm, const Workspace& ws, const void* Wd,
                             const void* Wds, bool bf16, int n_sms, cudaStream_t st) {
  int n_clusters = (2 * n_sms + kCluster - 1) / kCluster;
  if (n_clusters < 1) n_clusters = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_clusters * kCluster);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (bf16)
    return cudaLaunchKernelEx(&cfg, down_gemv_kernel<__nv_bfloat16, 4>, dm, ws,
                              static_cast<const __nv_bfloat16*>(Wd),
                              static_cast<const __nv_bfloat16*>(Wds));
  return cudaLaunchKernelEx(&cfg, down_gemv_kernel<float, 8>, dm, ws,
                            static_cast<const float*>(Wd), static_cast<const float*>(Wds));
}

}  // namespace moe
