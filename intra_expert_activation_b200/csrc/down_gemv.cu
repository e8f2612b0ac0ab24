// Down projection on CUDA cores for expert token groups with few tokens
// (decode): stream only the W_down rows in the group's active-neuron union
// and multiply them by the tokens' h values.
//
// This is the low-batch side of the pages' batch-size switch [gist.science
// EN "Uncovering Intra-expert Activation Sparsity for Efficient
// Mixture-of-Expert Model Execution", Technical Summary > Methodology >
// System Implementation in vLLM > "Dynamic Switching"]: with one to a few
// tokens per expert the down projection is a matrix-vector product whose
// cost is the bytes of the rows it reads ["Fused Up-Down Projection": only
// the active neurons' weights are fetched].
//
// Work: a unit is (group, pass of up to MT tokens); its neuron range is cut
// into splits of whole union-bitmap words, and a work item is one split of
// one unit over all d_model columns, described by a GemvItem the router
// wrote. One CTA per SM: 16 streaming warps and one scheduler warp. The
// scheduler takes the next item from an atomic queue and compacts its
// union-bitmap words into an ordered row list (double-buffered) while the
// streaming warps work on the current item, so items are balanced
// dynamically and their set-up is hidden. Each streaming warp owns one
// 512-byte column slice and streams the item's rows through its own ring of
// shared-memory stages with cp.async: per row 16 bytes of W_down per lane and
// the tokens' h values (one lane), kStages x kBatch rows in flight per warp
// with no registers held by data in flight; landed segments are multiplied
// by h with packed fp32x2 FMAs. An item that is a whole unit stores its
// result into Y[slot][columns]; a split adds its partial into Y (zeroed by the
// router) with vector fp32 atomics, so the splits of a unit are summed in
// arrival order: results agree to fp32 rounding, not bitwise, between runs on
// this path.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kStreamWarps = 16;
constexpr int kThreads = (kStreamWarps + 1) * 32;  // + the scheduler warp
constexpr int kBatch = 8;    // rows per stage
constexpr int kStages = 3;   // stages per warp ring
constexpr int kHBytes = 32;  // h bytes kept per row (MT x element: 8 for bf16, 32 for fp32)
constexpr int kStageBytes = kBatch * 512 + kBatch * kHBytes;
constexpr int kWarpRing = kStages * kStageBytes;  // bytes per warp ring

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// Packed pair of fp32 values and d = a * b + d on both lanes of the pair.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ void fma2(uint64_t& d, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

// A landed 16-byte weight segment as packed fp32 pairs.
template <typename TW>
struct Seg;
template <>
struct Seg<__nv_bfloat16> {
  static constexpr int VEC = 8, NP = 4;
  __device__ static void pairs(const uint4& u, uint64_t (&w)[4]) {
    const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)  // bf16 pair -> (low << 16, high & 0xffff0000) as fp32
      w[i] = pack2(__uint_as_float(q[i] << 16), __uint_as_float(q[i] & 0xffff0000u));
  }
};
template <>
struct Seg<float> {
  static constexpr int VEC = 4, NP = 2;
  __device__ static void pairs(const uint4& u, uint64_t (&w)[2]) {
    w[0] = pack2(__uint_as_float(u.x), __uint_as_float(u.y));
    w[1] = pack2(__uint_as_float(u.z), __uint_as_float(u.w));
  }
};

// Token t's h of a row as landed in the ring, broadcast to a packed pair.
template <typename TW>
__device__ __forceinline__ uint64_t h_pair(const uint8_t* p, int t) {
  float h;
  if constexpr (sizeof(TW) == 2)
    h = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(p)[t]) << 16);
  else
    h = reinterpret_cast<const float*>(p)[t];
  return pack2(h, h);
}

struct Staged {
  GemvItem it;
  int item;  // index, or >= n_items when the queue is empty
  int n;     // rows
};

// One streaming warp: rows of the staged item through its cp.async ring,
// MTE tokens accumulated in packed fp32 pairs; stores or adds mt results.
template <typename TW, int MT, int MTE>
__device__ __forceinline__ void stream_rows(const char* Wb, const char* hb, float* y, int d,
                                            uint32_t w_stride, uint32_t h_stride,
                                            const int* srow, int n, int rstride, int mt,
                                            bool whole,
                                            uint8_t* ring, uint32_t ring_s, int lane) {
  constexpr int NP = Seg<TW>::NP;
  constexpr int HB = MT * static_cast<int>(sizeof(TW));
  const int nb = (n + kBatch - 1) / kBatch;
  auto issue = [&](int b) {
    if (b < nb) {
      const uint32_t st = ring_s + (b % kStages) * kStageBytes;
      const int q0 = b * kBatch;
      const int cnt = min(kBatch, n - q0);
#pragma unroll
      for (int r = 0; r < kBatch; ++r) {
        if (r < cnt) {
          const uint32_t j = static_cast<uint32_t>(srow[(q0 + r) * rstride]);
          cp_async16(st + r * 512 + lane * 16, Wb + j * w_stride);
          const uint32_t hdst = st + kBatch * 512 + r * kHBytes;
          if constexpr (HB == 8) {
            if (lane == 0) cp_async8(hdst, hb + j * h_stride);
          } else {
            if (lane * 16 < HB) cp_async16(hdst + lane * 16, hb + j * h_stride + lane * 16);
          }
        }
      }
    }
    cp_async_commit();
  };
  uint64_t acc[MTE][NP];
#pragma unroll
  for (int t = 0; t < MTE; ++t)
#pragma unroll
    for (int v = 0; v < NP; ++v) acc[t][v] = 0ull;
#pragma unroll
  for (int b = 0; b < kStages - 1; ++b) issue(b);
  for (int b = 0; b < nb; ++b) {
    issue(b + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncwarp();  // the h slots were copied by other lanes
    const uint8_t* st = ring + (b % kStages) * kStageBytes;
    const int cnt = min(kBatch, n - b * kBatch);
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      if (r < cnt) {
        uint64_t w[NP];
        Seg<TW>::pairs(*reinterpret_cast<const uint4*>(st + r * 512 + lane * 16), w);
        const uint8_t* hp = st + kBatch * 512 + r * kHBytes;
#pragma unroll
        for (int t = 0; t < MTE; ++t) {
          const uint64_t h2 = h_pair<TW>(hp, t);
#pragma unroll
          for (int v = 0; v < NP; ++v) fma2(acc[t][v], h2, w[v]);
        }
      }
    }
    __syncwarp();  // every lane has read the stage before it is refilled
  }
  cp_async_wait<0>();
#pragma unroll
  for (int t = 0; t < MTE; ++t) {
    if (t < mt) {
      float* yt = y + static_cast<size_t>(t) * d;
#pragma unroll
      for (int v = 0; v < NP; v += 2) {
        const float2 a = unpack2(acc[t][v]), c = unpack2(acc[t][v + 1]);
        if (whole)
          *reinterpret_cast<float4*>(yt + 2 * v) = make_float4(a.x, a.y, c.x, c.y);
        else
          red_add_v4(yt + 2 * v, a.x, a.y, c.x, c.y);
      }
    }
  }
}

template <typename TW, int MT>
__global__ void __launch_bounds__(kThreads, 1)
    down_gemv_kernel(Dims dm, Workspace ws, const TW* __restrict__ Wd,
                     const TW* __restrict__ Wds) {
  constexpr int VEC = Seg<TW>::VEC;
  constexpr int SW = 32 * VEC;  // columns per slice: one 512-byte row segment
  static_assert(MT * sizeof(TW) <= kHBytes, "h slot");
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* rings = smem;                                             // [16][kWarpRing]
  int* srow = reinterpret_cast<int*>(smem + kStreamWarps * kWarpRing);  // [2][kGemvRowsMax]
  __shared__ Staged staged[2];

  grid_dep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = dm.d;
  const int n_slices = d / SW;
  const int n_phase = n_slices >= kStreamWarps ? 1 : kStreamWarps / n_slices;  // warps per slice
  const int n_tasks = n_slices * n_phase;
  const int n_items = __ldcg(ws.meta + kMetaGemvItems);
  const size_t ld = static_cast<size_t>(dm.slots_total);
  const TW* ht = static_cast<const TW*>(ws.ht);

  // scheduler warp: take the next item and stage its rows into buffer b
  auto fetch = [&](int b) {
    int idx = 0;
    if (lane == 0) idx = atomicAdd(ws.meta + kMetaGemvNext, 1);
    idx = __shfl_sync(0xffffffffu, idx, 0);
    if (idx >= n_items) {
      if (lane == 0) staged[b].item = n_items;
      return;
    }
    const GemvItem it = ws.gemv_items[idx];
    const int nw = it.w1 - it.w0;  // <= kGemvWordsMax <= 32
    const uint32_t bits =
        lane < nw ? __ldcg(ws.union_bits + static_cast<size_t>(it.g) * dm.fw + it.w0 + lane) : 0u;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int* rows = srow + b * kGemvRowsMax;
    int pos = incl - c;
    uint32_t bb = bits;
    const int base = 32 * (it.w0 + lane);
    while (bb) {
      rows[pos++] = base + __ffs(bb) - 1;
      bb &= bb - 1;
    }
    if (lane == 31) {
      staged[b].it = it;
      staged[b].n = incl;
      staged[b].item = idx;
      atomicAdd(ws.counters + kCntDownRows, static_cast<unsigned long long>(incl));
    }
  };

  if (warp == kStreamWarps) fetch(0);
  __syncthreads();
  for (int cur = 0;; cur ^= 1) {
    if (staged[cur].item >= n_items) break;
    if (warp == kStreamWarps) {
      fetch(cur ^ 1);
    } else {
      const GemvItem it = staged[cur].it;
      const int n = staged[cur].n;
      const int* rows = srow + cur * kGemvRowsMax;
      const bool shared = it.expert >= dm.E;
      const int F_e = shared ? dm.Fs : dm.F;
      const TW* Wbase = shared ? Wds + static_cast<size_t>(it.expert - dm.E) * F_e * d
                               : Wd + static_cast<size_t>(it.expert) * F_e * d;
      float* y = ws.y + static_cast<size_t>(it.slot) * d;
      const bool whole = it.whole && n_phase == 1;
      const uint32_t w_stride = d * sizeof(TW), h_stride = ld * sizeof(TW);
      uint8_t* ring = rings + warp * kWarpRing;
      const uint32_t ring_s = smem_u32(ring);
      for (int task = warp; task < n_tasks; task += kStreamWarps) {
        const int slice = task % n_slices, phase = task / n_slices;
        const int col = slice * SW + lane * VEC;
        // this warp's rows: phase, phase + n_phase, ...
        const int* wrows = rows + phase;
        const int nq = n > phase ? (n - phase + n_phase - 1) / n_phase : 0;
        const char* Wb = reinterpret_cast<const char*>(Wbase + col);
        const char* hb = reinterpret_cast<const char*>(ht + it.slot);
        if (it.mt <= 1)
          stream_rows<TW, MT, 1>(Wb, hb, y + col, d, w_stride, h_stride, wrows, nq, n_phase,
                                 it.mt, whole, ring, ring_s, lane);
        else if (it.mt <= 2 && MT > 2)
          stream_rows<TW, MT, 2>(Wb, hb, y + col, d, w_stride, h_stride, wrows, nq, n_phase,
                                 it.mt, whole, ring, ring_s, lane);
        else
          stream_rows<TW, MT, MT>(Wb, hb, y + col, d, w_stride, h_stride, wrows, nq, n_phase,
                                  it.mt, whole, ring, ring_s, lane);
      }
    }
    __syncthreads();
  }
}

}  // namespace

size_t down_gemv_smem_bytes(bool) {
  return static_cast<size_t>(kStreamWarps) * kWarpRing + 2 * sizeof(int) * kGemvRowsMax;
}

cudaError_t launch_down_gemv(const Dims& dm, const Workspace& ws, const void* Wd,
                             const void* Wds, bool bf16, int n_sms, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(down_gemv_kernel<__nv_bfloat16, kGemvTokens>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)down_gemv_smem_bytes(true));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(down_gemv_kernel<float, 8>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)down_gemv_smem_bytes(false));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = n_sms;  // one CTA per SM
  if (bf16)
    return launch_k(down_gemv_kernel<__nv_bfloat16, kGemvTokens>, grid, kThreads,
                    down_gemv_smem_bytes(true), st, dm, ws,
                    static_cast<const __nv_bfloat16*>(Wd), static_cast<const __nv_bfloat16*>(Wds));
  return launch_k(down_gemv_kernel<float, 8>, grid, kThreads, down_gemv_smem_bytes(false), st,
                  dm, ws, static_cast<const float*>(Wd), static_cast<const float*>(Wds));
}

}  // namespace moe
