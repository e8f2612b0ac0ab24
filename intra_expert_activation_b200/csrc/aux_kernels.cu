// Small kernels between the big ones:
//  union_scan   (forced gathered tensor-core mode only) per expert token
//               group: mark groups of <= kGatherMaxTokens tokens for the
//               gathered path and count the rows the down projection reads
//               (the tensor-core kernel walks the union bitmaps itself)
//               [gist.science EN "Uncovering Intra-expert Activation
//               Sparsity for Efficient Mixture-of-Expert Model Execution",
//               Technical Summary > Methodology > System Implementation in
//               vLLM > "Fused Up-Down Projection"].
//  combine      out[t] = sum_i w[t,i] * Y[slot(t,i)] + sum_s Y[shared slot(s,t)],
//               in a fixed order.
//  debug_gather routing and active bitmaps of the last forward in pair order.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kScanThreads = 256;
__global__ void __launch_bounds__(kScanThreads) union_scan_kernel(Dims dm, Workspace ws) {
  grid_dep_wait();
  const int n_groups = __ldcg(ws.meta + kMetaGroups);
  for (int g = blockIdx.x * kScanThreads + threadIdx.x; g < n_groups;
       g += gridDim.x * kScanThreads) {
    // gathered rows for groups of <= kGatherMaxTokens tokens, all rows above;
    // the union's rows were counted by the gate/up epilogue
    const Group gr = ws.groups[g];
    const int F_e = gr.expert >= dm.E ? dm.Fs : dm.F;
    const int cnt = __ldcg(ws.union_cnt + g);
    const int path = gr.m <= kGatherMaxTokens ? kPathTcGather : kPathTcAll;
    ws.group_path[g] = path;
    atomicAdd(ws.counters + kCntDownRows,
              static_cast<unsigned long long>(path == kPathTcAll ? F_e : cnt));
    if (path == kPathTcGather) atomicAdd(ws.counters + kCntTcGather, 1ull);
  }
}

template <typename TX>
__device__ __forceinline__ void store4(TX* p, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
  union { __nv_bfloat162 b[2]; uint2 u; } pk;
  pk.b[0] = __floats2bfloat162_rn(v.x, v.y);
  pk.b[1] = __floats2bfloat162_rn(v.z, v.w);
  *reinterpret_cast<uint2*>(p) = pk.u;
}

template <typename TX>
__global__ void __launch_bounds__(256) combine_kernel(Dims dm, Workspace ws, TX* out, int nb) {
  grid_dep_wait();
  // CTA = (token, block of blockDim x 4 columns): every column of a token is
  // in flight at once, and each thread's k + S row loads are issued together
  const int t = blockIdx.x / nb;
  const int c = ((blockIdx.x % nb) * blockDim.x + threadIdx.x) * 4;
  const int d = dm.d, k = dm.k;
  __shared__ int slot[16];
  __shared__ float w[16];
  if (threadIdx.x < k) {
    int s = __ldcg(ws.slot_of + t * k + threadIdx.x);
    if (!moe_in_bounds(ws.status, s >= 0 && s < dm.slots_routed)) s = 0;
    slot[threadIdx.x] = s;
    w[threadIdx.x] = __ldcg(ws.topk_w + t * k + threadIdx.x);
  }
  __syncthreads();
  if (c >= d) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int i = 0; i < k; ++i) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(ws.y + static_cast<size_t>(slot[i]) * d + c));
    acc.x = fmaf(w[i], v.x, acc.x);
    acc.y = fmaf(w[i], v.y, acc.y);
    acc.z = fmaf(w[i], v.z, acc.z);
    acc.w = fmaf(w[i], v.w, acc.w);
  }
  for (int s = 0; s < dm.S; ++s) {
    const size_t srow = static_cast<size_t>(dm.slots_routed + s * dm.T_pad + t);
    const float4 v = __ldcg(reinterpret_cast<const float4*>(ws.y + srow * d + c));
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  store4<TX>(out + static_cast<size_t>(t) * d + c, acc);
}

__global__ void debug_gather_kernel(Dims dm, Workspace ws, int32_t* topk_idx, float* topk_w,
                                    uint32_t* bits, uint32_t* bits_shared) {
  grid_dep_wait();
  const int P = dm.T * dm.k;
  const int fwr = (dm.F + 31) / 32, fws = (dm.Fs + 31) / 32;
  const int stride = gridDim.x * blockDim.x;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < P; i += stride) {
    if (topk_idx) topk_idx[i] = ws.topk_idx[i];
    if (topk_w) topk_w[i] = ws.topk_w[i];
  }
  if (bits && ws.act_bits) {
    for (long long i = blockIdx.x * blockDim.x + threadIdx.x; i < (long long)P * fwr; i += stride) {
      const int p = static_cast<int>(i / fwr), w = static_cast<int>(i % fwr);
      bits[i] = ws.act_bits[static_cast<size_t>(ws.slot_of[p]) * dm.fw + w];
    }
  }
  if (bits_shared && ws.act_bits && dm.S > 0) {
    const long long n = (long long)dm.S * dm.T * fws;
    for (long long i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
      const int w = static_cast<int>(i % fws);
      const long long st = i / fws;
      const int t = static_cast<int>(st % dm.T), s = static_cast<int>(st / dm.T);
      const size_t slot = static_cast<size_t>(dm.slots_routed + s * dm.T_pad + t);
      bits_shared[i] = ws.act_bits[slot * dm.fw + w];
    }
  }
}

#if MOE_CHECK
// Checked build only: exercises the kernels' bounded waits with an arrival
// that never comes. which = 0: an mbarrier that expects one arrival, waited
// on by warp 0 through warp_wait; which = 1: a flag in global memory that
// nothing sets, waited on through wait_flag. Either wait gives up after
// `limit` probes, records MOE_ERR_DEVICE_TIMEOUT in the status word and the
// kernel returns.
__device__ int g_flag_never_set = 0;
__global__ void wait_timeout_kernel(int* status, uint32_t limit, int which) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (which == 0) {
    if (threadIdx.x < 32) warp_wait(&bar, 0, &abort_flag, status, 0, limit);
  } else if (threadIdx.x == 0) {
    wait_flag(&g_flag_never_set, &abort_flag, status, limit);
  }
}
#endif

}  // namespace

#if MOE_CHECK
cudaError_t launch_wait_timeout(int* status, uint32_t limit, int which, cudaStream_t st) {
  wait_timeout_kernel<<<1, 64, 0, st>>>(status, limit, which);
  return cudaGetLastError();
}
#endif

cudaError_t launch_union_scan(const Dims& dm, const Workspace& ws, cudaStream_t st) {
  return launch_k(union_scan_kernel, (dm.groups_max + kScanThreads - 1) / kScanThreads,
                  kScanThreads, 0, st, dm, ws);
}

cudaError_t launch_combine(const Dims& dm, const Workspace& ws, void* out, bool bf16,
                           cudaStream_t st) {
  const int threads = dm.d / 4 >= 256 ? 256 : ((dm.d / 4 + 31) / 32) * 32;
  const int nb = (dm.d / 4 + threads - 1) / threads;  // column blocks per token
  const int grid = dm.T * nb;
  if (bf16)
    return launch_k(combine_kernel<__nv_bfloat16>, grid, threads, 0, st, dm, ws,
                    static_cast<__nv_bfloat16*>(out), nb);
  return launch_k(combine_kernel<float>, grid, threads, 0, st, dm, ws, static_cast<float*>(out),
                  nb);
}

cudaError_t launch_debug_gather(const Dims& dm, const Workspace& ws, int32_t* topk_idx,
                                float* topk_w, uint32_t* bits, uint32_t* bits_shared,
                                cudaStream_t st) {
  debug_gather_kernel<<<256, 256, 0, st>>>(dm, ws, topk_idx, topk_w, bits, bits_shared);
  return cudaGetLastError();
}

}  // namespace moe
