// moe_sparse_route_noalloc: the layer's routing step (logits, softmax, top-k,
// stable grouping of the (token, expert) pairs by expert) for callers that
// must not allocate device memory, for example plug-ins that live inside
// another framework's fixed memory plan, or serving loops that reserve all
// device memory up front and treat a later allocation as a failure. It
// computes what the forward's router computes, into caller buffers, and keeps
// its scratch (per-CTA expert histograms, per-pair ranks, a completion
// ticket) in one file-scope device array instead of a context workspace.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "kernels.h"
#include "topk.cuh"
#include "moe_sparse.h"

namespace moe {
void set_last_error(const std::string& msg);  // moe_sparse.cu
}

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxE = 256;
constexpr int kMaxTokensNA = 4096;
constexpr int kMaxK = 16;
constexpr size_t kScratchBytes = size_t(1) << 20;  // 1 MiB on every device that loads the library
constexpr int kCtlBytes = 256;                     // ticket word + padding

// Scratch of moe_sparse_route_noalloc. In host code this name is a host-side
// stand-in: the kernel receives the device address found with
// cudaGetSymbolAddress at set-up.
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

int tokens_per_cta(int T) { return T <= 256 ? 2 : 16; }

struct NaArgs {
  const void* x;
  const void* Wr;
  const float* bias;
  int T, d, E, k, renorm, tpc;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* offsets;  // [E+1]
  int32_t* slot_of;  // [T*k]
  int32_t* perm;     // [T*k]
  unsigned char* scratch;
};

template <typename TX>
__device__ __forceinline__ void load8(const TX* p, float (&f)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(b[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <typename TX>
__global__ void __launch_bounds__(kThreads) route_noalloc_kernel(NaArgs a) {
  __shared__ float lg[16][kMaxE + 1];
  __shared__ int sel[16 * kMaxK];
  __shared__ int wcnt[kWarps][kMaxE];
  __shared__ int base_s[kMaxE + 1];
  __shared__ int is_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, d = a.d, k = a.k, T = a.T;
  const int tok0 = blockIdx.x * a.tpc;
  const int tb = min(a.tpc, T - tok0);
  int* ticket = reinterpret_cast<int*>(a.scratch);
  int* hist = reinterpret_cast<int*>(a.scratch + kCtlBytes);  // [n_cta][E]
  int* rank = hist + static_cast<size_t>(gridDim.x) * E;      // [T*k]
  const TX* x = static_cast<const TX*>(a.x);
  const TX* Wr = static_cast<const TX*>(a.Wr);

  // logits: warp tasks (token, expert), lanes over d in 8-element chunks
  for (int task = warp; task < tb * E; task += kWarps) {
    const int t = task / E, e = task % E;
    const TX* xr = x + static_cast<size_t>(tok0 + t) * d;
    const TX* wr = Wr + static_cast<size_t>(e) * d;
    float acc = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      float xv[8], wv[8];
      load8<TX>(xr + c, xv);
      load8<TX>(wr + c, wv);
#pragma unroll
      for (int v = 0; v < 8; ++v) acc = fmaf(xv[v], wv[v], acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) lg[t][e] = acc + (a.bias ? a.bias[e] : 0.f);
  }
  for (int i = tid; i < kWarps * kMaxE; i += kThreads) (&wcnt[0][0])[i] = 0;
  __syncthreads();

  // top-k per token: the k largest logits, ties to the lower expert index
  // (NaN logits rank as -inf; the ids are distinct and in [0, E))
  for (int t = warp; t < tb; t += kWarps) {
    const moe::TopkResult r = moe::topk_warp(lg[t], E, k, lane);
    if (lane < k) {
      const int tok = tok0 + t;
      a.topk_idx[tok * k + lane] = r.my_e;
      a.topk_w[tok * k + lane] = a.renorm ? r.my_p / r.psum : r.my_p;
      sel[t * k + lane] = r.my_e;
    }
  }
  __syncthreads();

  // stable rank of each of the CTA's pairs among its pairs of the same expert
  const int np = tb * k;
  const int e = tid < np ? sel[tid] : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int r0 = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && r0 == 0) wcnt[warp][e] = __popc(peers);
  __syncthreads();
  if (e >= 0) {
    int r = r0;
    for (int w = 0; w < warp; ++w) r += wcnt[w][e];
    rank[tok0 * k + tid] = r;
  }
  for (int x2 = tid; x2 < E; x2 += kThreads) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) c += wcnt[w][x2];
    hist[static_cast<size_t>(blockIdx.x) * E + x2] = c;
  }

  // the last CTA to finish lays out the slots for the whole batch
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    is_last = atomicAdd(ticket, 1) == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const int n_cta = gridDim.x;
  // per expert: exclusive scan over CTAs (hist becomes base offsets)
  for (int ex = tid; ex < E; ex += kThreads) {
    int run = 0;
    for (int c = 0; c < n_cta; ++c) {
      int* h = hist + static_cast<size_t>(c) * E + ex;
      const int v = __ldcg(h);
      *h = run;
      run += v;
    }
    base_s[ex] = run;  // count of expert ex
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0;
    for (int ex = 0; ex < E; ++ex) {
      const int c = base_s[ex];
      base_s[ex] = off;
      a.offsets[ex] = off;
      off += c;
    }
    a.offsets[E] = off;
    *ticket = 0;  // ready for the next call
  }
  __syncthreads();
  __threadfence();
  const int P = T * k;
  for (int p = tid; p < P; p += kThreads) {
    const int ex = __ldcg(a.topk_idx + p);
    const int c = (p / k) / a.tpc;
    const int slot = base_s[ex] + __ldcg(hist + static_cast<size_t>(c) * E + ex) + __ldcg(rank + p);
    a.slot_of[p] = slot;
    a.perm[slot] = p / k;
  }
}

std::mutex g_mu;
void* g_scratch_ptr[256] = {};  // device address of g_route_scratch, per device ordinal

moe_status fail(moe_status s, const std::string& msg) {
  moe::set_last_error(msg);
  return s;
}

}  // namespace

extern "C" MOE_API moe_status moe_sparse_route_noalloc(
    const void* x, int32_t T, int32_t d_model, const void* W_router, const float* router_bias,
    int32_t n_experts, int32_t top_k, int32_t renormalize, int32_t dtype, int32_t* topk_idx,
    float* topk_w, int32_t* expert_offsets, int32_t* slot_of, int32_t* perm, void* stream) {
  if (dtype != MOE_BF16 && dtype != MOE_F32) return fail(MOE_ERR_INVALID, "dtype must be MOE_F32 or MOE_BF16");
  if (T < 0) return fail(MOE_ERR_INVALID, "T < 0");
  if (T > kMaxTokensNA)
    return fail(MOE_ERR_UNSUPPORTED, "moe_sparse_route_noalloc: T > 4096 exceeds its fixed scratch");
  if (n_experts < 1 || n_experts > kMaxE)
    return fail(MOE_ERR_UNSUPPORTED, "moe_sparse_route_noalloc: n_experts must be in 1..256");
  if (top_k < 1 || top_k > n_experts || top_k > kMaxK)
    return fail(MOE_ERR_INVALID, "top_k must be in 1..min(n_experts, 16)");
  const int dmod = dtype == MOE_BF16 ? 256 : 128;
  if (d_model <= 0 || d_model % dmod)
    return fail(MOE_ERR_UNSUPPORTED, "d_model must be a positive multiple of 256 (bf16) or 128 (fp32)");
  if (!expert_offsets) return fail(MOE_ERR_INVALID, "expert_offsets is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (n_experts + 1), st);
    return e == cudaSuccess ? MOE_OK : fail(MOE_ERR_CUDA, cudaGetErrorString(e));
  }
  if (!x || !W_router || !topk_idx || !topk_w || !slot_of || !perm)
    return fail(MOE_ERR_INVALID, "NULL pointer");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(W_router)) & 15u)
    return fail(MOE_ERR_INVALID, "x and W_router must be 16-byte aligned");

  const int tpc = tokens_per_cta(T);
  const int n_cta = (T + tpc - 1) / tpc;
  const size_t need = kCtlBytes + sizeof(int) * (static_cast<size_t>(n_cta) * n_experts +
                                                 static_cast<size_t>(T) * top_k);
  if (need > kScratchBytes)
    return fail(MOE_ERR_UNSUPPORTED, "moe_sparse_route_noalloc: batch exceeds its fixed scratch");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 256) return fail(MOE_ERR_CUDA, "cudaGetDevice failed");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {  // set-up, once per device, with that device current
      e = cudaGetSymbolAddress(&g_scratch_ptr[dev], g_route_scratch);
      if (e != cudaSuccess) {
        g_scratch_ptr[dev] = nullptr;
        return fail(MOE_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      }
    }
    scratch = g_scratch_ptr[dev];
  }
  // the completion ticket must start at zero
  e = cudaMemsetAsync(scratch, 0, kCtlBytes, st);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, cudaGetErrorString(e));

  NaArgs a;
  a.x = x;
  a.Wr = W_router;
  a.bias = router_bias;
  a.T = T;
  a.d = d_model;
  a.E = n_experts;
  a.k = top_k;
  a.renorm = renormalize ? 1 : 0;
  a.tpc = tpc;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.offsets = expert_offsets;
  a.slot_of = slot_of;
  a.perm = perm;
  a.scratch = static_cast<unsigned char*>(scratch);
  if (dtype == MOE_BF16)
    route_noalloc_kernel<__nv_bfloat16><<<n_cta, kThreads, 0, st>>>(a);
  else
    route_noalloc_kernel<float><<<n_cta, kThreads, 0, st>>>(a);
  e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : fail(MOE_ERR_CUDA, cudaGetErrorString(e));
}
