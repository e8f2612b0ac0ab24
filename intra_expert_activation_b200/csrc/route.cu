// Router: logits, softmax over all experts, top-k (+ renormalisation), then a
// deterministic stable counting sort of the routed (token, expert) pairs into
// per-expert slot ranges and expert token groups. The pages keep the dense
// model's router as it is [gist.science EN "Uncovering Intra-expert
// Activation Sparsity for Efficient Mixture-of-Expert Model Execution",
// Technical Summary > Methodology > System Implementation in vLLM].
//
// route_kernel: one CTA per 32 tokens. Logits are fp32 dot products over
// shared-memory tiles of x and W_router (sequential in d, so every call gives
// the same bits). One warp per token then picks the top-k by logit (equal
// logits: lower expert index), and the softmax weights. The last CTA to
// finish (atomic ticket after a fence) runs the scan for the whole batch.
//
// permute_kernel: X_perm[slot] = x[perm[slot]] (zero rows for padding slots).
#include "common.cuh"

namespace moe {

namespace {

constexpr int kRouteTokens = 32;
constexpr int kRouteThreads = 256;
constexpr int kRouteChunk = 32;
constexpr int kMaxExperts = 256;
constexpr int kPad = kRouteChunk + 1;

template <typename TX>
__device__ __forceinline__ float ldf(const TX* p) {
  return to_f32<TX>(*p);
}

// Total order used by the top-k: larger logit first, then lower index.
__device__ __forceinline__ bool better(float va, int ea, float vb, int eb) {
  return va > vb || (va == vb && ea < eb);
}

__device__ void route_scan(const Dims& dm, const Workspace& ws, int* smem_i) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int E = dm.E, k = dm.k, T = dm.T;
  const int P = T * k;
  int* cnt = smem_i;                     // [E]
  int* poff = cnt + kMaxExperts;         // [E+1]
  int* run = poff + kMaxExperts + 1;     // [E]
  int* wcnt = run + kMaxExperts;         // [8][E]

  for (int e = tid; e < E; e += blockDim.x) { cnt[e] = 0; run[e] = 0; }
  for (int i = tid; i < 8 * kMaxExperts; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  for (int p = tid; p < P; p += blockDim.x) atomicAdd(&cnt[__ldcg(ws.topk_idx + p)], 1);
  __syncthreads();

  if (tid == 0) {
    int touched = 0;
    poff[0] = 0;
    for (int e = 0; e < E; ++e) {
      const int me = cnt[e];
      touched += me > 0;
      poff[e + 1] = poff[e] + (me + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
    }
    int ng = 0;
    for (int e = 0; e < E; ++e) {
      const int me = cnt[e];
      if (me == 0) continue;
      const int n_g = (me + kGroupMax - 1) / kGroupMax;
      int gsz = (me + n_g - 1) / n_g;
      gsz = (gsz + 63) / 64 * 64;
      for (int g = 0; g * gsz < me && ng < dm.groups_max; ++g) {
        Group gr;
        gr.expert = e;
        gr.slot0 = poff[e] + g * gsz;
        gr.m = min(gsz, me - g * gsz);
        gr.xrow0 = gr.slot0;
        ws.groups[ng++] = gr;
      }
    }
    ws.meta[kMetaRoutedGroups] = ng;
    for (int s = 0; s < dm.S; ++s) {
      const int n_g = (T + kGroupMax - 1) / kGroupMax;
      int gsz = (T + n_g - 1) / n_g;
      gsz = (gsz + 63) / 64 * 64;
      for (int g = 0; g * gsz < T && ng < dm.groups_max; ++g) {
        Group gr;
        gr.expert = E + s;
        gr.slot0 = dm.slots_routed + s * dm.T_pad + g * gsz;
        gr.m = min(gsz, T - g * gsz);
        gr.xrow0 = g * gsz;
        ws.groups[ng++] = gr;
      }
    }
    ws.meta[kMetaGroups] = ng;
    ws.meta[kMetaSlotsUsed] = poff[E];
    ws.meta[kMetaExpertsTouched] = touched;
    ws.meta[kMetaGemvCount] = 0;
    ws.meta[kMetaTcCount] = 0;
  }
  __syncthreads();

  // padding slots of each expert's range hold no token
  for (int e = warp; e < E; e += blockDim.x / 32)
    for (int s = poff[e] + cnt[e] + lane; s < poff[e + 1]; s += 32) ws.perm[s] = -1;

  // stable scatter, pairs in (token, choice) order
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < P; base += blockDim.x) {
    const int p = base + tid;
    const int e = p < P ? __ldcg(ws.topk_idx + p) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt_mask);
    if (e >= 0 && rank == 0) wcnt[warp * kMaxExperts + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int off = run[e] + rank;
      for (int w = 0; w < warp; ++w) off += wcnt[w * kMaxExperts + e];
      const int slot = poff[e] + off;
      ws.perm[slot] = p / k;
      ws.slot_of[p] = slot;
    }
    __syncthreads();
    for (int e2 = tid; e2 < E; e2 += blockDim.x) {
      int tot = 0;
      for (int w = 0; w < (int)(blockDim.x / 32); ++w) {
        tot += wcnt[w * kMaxExperts + e2];
        wcnt[w * kMaxExperts + e2] = 0;
      }
      run[e2] += tot;
    }
    __syncthreads();
  }

  if (tid < kCntWords) ws.counters[tid] = 0ull;
  __syncthreads();
  if (tid == 0) {
    ws.counters[kCntRoutedH] = (unsigned long long)P * (unsigned long long)dm.F;
    ws.counters[kCntSharedH] =
        (unsigned long long)dm.S * (unsigned long long)T * (unsigned long long)dm.Fs;
    ws.meta[kMetaDone] = 0;  // ticket counter for the next forward
  }
}

template <typename TX>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(Dims dm, Workspace ws, const TX* x,
                                                              const TX* Wr, const float* bias) {
  __shared__ float xs[kRouteTokens * kPad];
  __shared__ float wsm[kMaxExperts * kPad];  // reused for logits and the scan
  __shared__ int is_last;

  const int tid = threadIdx.x;
  const int tok0 = blockIdx.x * kRouteTokens;
  const int E = dm.E, d = dm.d, T = dm.T, k = dm.k;
  const int tt = tid >> 3, eg = tid & 7;
  const int nq = (E + 7) / 8;

  float acc[kMaxExperts / 8];
#pragma unroll
  for (int q = 0; q < kMaxExperts / 8; ++q) acc[q] = 0.f;

  for (int d0 = 0; d0 < d; d0 += kRouteChunk) {
    for (int i = tid; i < kRouteTokens * kRouteChunk; i += kRouteThreads) {
      const int t = i / kRouteChunk, c = i % kRouteChunk;
      const int tok = tok0 + t;
      xs[t * kPad + c] = tok < T ? ldf(x + (size_t)tok * d + d0 + c) : 0.f;
    }
    for (int i = tid; i < E * kRouteChunk; i += kRouteThreads) {
      const int e = i / kRouteChunk, c = i % kRouteChunk;
      wsm[e * kPad + c] = ldf(Wr + (size_t)e * d + d0 + c);
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kRouteChunk; ++c) {
      const float xv = xs[tt * kPad + c];
#pragma unroll
      for (int q = 0; q < kMaxExperts / 8; ++q)
        if (q < nq) acc[q] = fmaf(xv, wsm[(eg + 8 * q) * kPad + c], acc[q]);
    }
    __syncthreads();
  }

  // logits [32][E+1] in the (now free) W tile
  float* lg = wsm;
  const int lgp = E + 1;
#pragma unroll
  for (int q = 0; q < kMaxExperts / 8; ++q) {
    const int e = eg + 8 * q;
    if (q < nq && e < E) lg[tt * lgp + e] = acc[q] + (bias ? bias[e] : 0.f);
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t < kRouteTokens; t += kRouteThreads / 32) {
    const int tok = tok0 + t;
    if (tok >= T) break;
    float v[kMaxExperts / 32];
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j) {
      const int e = lane + 32 * j;
      v[j] = e < E ? lg[t * lgp + e] : -INFINITY;
    }
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j) mx = fmaxf(mx, v[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float z = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j)
      if (lane + 32 * j < E) z += expf(v[j] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);

    int my_e = -1;
    float my_p = 0.f, psum = 0.f;
    for (int i = 0; i < k; ++i) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < kMaxExperts / 32; ++j) {
        const int e = lane + 32 * j;
        if (e < E && better(v[j], e, bv, be)) { bv = v[j]; be = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (better(ov, oe, bv, be)) { bv = ov; be = oe; }
      }
#pragma unroll
      for (int j = 0; j < kMaxExperts / 32; ++j)
        if (lane + 32 * j == be) v[j] = -INFINITY;
      const float p = expf(bv - mx) / z;
      psum += p;
      if (lane == i) { my_e = be; my_p = p; }
    }
    if (lane < k) {
      ws.topk_idx[tok * k + lane] = my_e;
      ws.topk_w[tok * k + lane] = dm.renorm ? my_p / psum : my_p;
    }
  }

  // the last CTA to finish builds the slot layout for the whole batch
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int ticket = atomicAdd(ws.meta + kMetaDone, 1);
    is_last = (ticket == (int)gridDim.x - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  route_scan(dm, ws, reinterpret_cast<int*>(wsm));
}

template <typename TX>
__global__ void __launch_bounds__(256) permute_kernel(Dims dm, Workspace ws, const TX* x) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= __ldcg(ws.meta + kMetaSlotsUsed)) return;
  const int tok = ws.perm[warp];
  constexpr int kVec = 16 / sizeof(TX);
  const int nv = dm.d / kVec;
  uint4* dst = reinterpret_cast<uint4*>(static_cast<TX*>(ws.xperm) + (size_t)warp * dm.d);
  if (tok < 0) {
    for (int i = lane; i < nv; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)tok * dm.d);
  for (int i = lane; i < nv; i += 32) dst[i] = __ldg(src + i);
}

}  // namespace

static_assert(sizeof(float) * kMaxExperts * kPad >=
                  sizeof(int) * (3 * kMaxExperts + 1 + 8 * kMaxExperts),
              "scan scratch must fit in the W tile");

cudaError_t launch_route(const Dims& dm, const Workspace& ws, const void* x, const void* Wr,
                         const float* bias, bool bf16, cudaStream_t st) {
  const int grid = (dm.T + kRouteTokens - 1) / kRouteTokens;
  if (bf16)
    route_kernel<__nv_bfloat16><<<grid, kRouteThreads, 0, st>>>(
        dm, ws, static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wr),
        bias);
  else
    route_kernel<float><<<grid, kRouteThreads, 0, st>>>(
        dm, ws, static_cast<const float*>(x), static_cast<const float*>(Wr), bias);
  return cudaGetLastError();
}

cudaError_t launch_permute(const Dims& dm, const Workspace& ws, const void* x, bool bf16,
                           cudaStream_t st) {
  const int rows = dm.slots_routed;
  const int grid = (rows + 7) / 8;
  if (bf16)
    permute_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(dm, ws,
                                                        static_cast<const __nv_bfloat16*>(x));
  else
    permute_kernel<float><<<grid, 256, 0, st>>>(dm, ws, static_cast<const float*>(x));
  return cudaGetLastError();
}

}  // namespace moe
