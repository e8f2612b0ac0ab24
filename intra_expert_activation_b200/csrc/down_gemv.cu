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
// Work: a unit is (group, pass of up to MT tokens); its union rows are cut
// into splits, and a work item is one split of one unit over all d_model
// columns. Persistent CTAs of 16 warps (one per SM) stride over the items. A
// CTA first stages the item's row ids and the tokens' h values in shared
// memory; then each warp owns one 512-byte column slice and streams the
// item's rows through its own ring of shared-memory stages with cp.async
// (16 bytes per lane per row; kStages x kBatch rows in flight per warp, with
// no registers held by data in flight), and multiplies each landed row
// segment by the tokens' h values into fp32 registers. Each lane copies and
// later reads back exactly its own 16 bytes, so a wait on the lane's own copy
// group is all the synchronisation the ring needs. An item that is a whole
// unit stores its result into Y[slot][columns]; a split adds its partial into
// Y (zeroed by the union scan) with vector fp32 atomics, so the splits of a
// unit are summed in arrival order: results agree to fp32 rounding, not
// bitwise, between runs on this path.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 8;    // rows per stage
constexpr int kStages = 3;   // stages per warp ring
constexpr int kWarpRing = kStages * kBatch * 32 * 16;  // bytes per warp ring

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

template <typename TW, int MT>
__global__ void __launch_bounds__(kThreads, 1)
    down_gemv_kernel(Dims dm, Workspace ws, const TW* __restrict__ Wd,
                     const TW* __restrict__ Wds) {
  constexpr int VEC = Vec<TW>::N;
  constexpr int SW = 32 * VEC;  // columns per slice: one 512-byte row segment
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* rings = smem;                                          // [kWarps][kWarpRing]
  int* srow = reinterpret_cast<int*>(smem + kWarps * kWarpRing);  // [kGemvRowsMax]
  float* sh = reinterpret_cast<float*>(srow + kGemvRowsMax);      // [kGemvRowsMax][MT]

  grid_dep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = dm.d;
  const int n_slices = d / SW;
  const int n_phase = n_slices >= kWarps ? 1 : kWarps / n_slices;  // warps per slice
  const int n_tasks = n_slices * n_phase;
  const int n_list = __ldcg(ws.meta + kMetaGemvCount);
  const int n_items = __ldcg(ws.meta + kMetaGemvItems);
  const int* item_off = ws.gemv_item_off;
  const int* unit_off = ws.gemv_item_off + dm.groups_max + 1;
  const size_t ld = static_cast<size_t>(dm.slots_total);
  const TW* ht = static_cast<const TW*>(ws.ht);
  uint8_t* ring = rings + warp * kWarpRing;
  const uint32_t ring_s = smem_u32(ring) + lane * 16;

  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    // listed group i with item_off[i] <= item < item_off[i + 1]
    int lo_i = 0, hi_i = n_list;
    while (hi_i - lo_i > 1) {
      const int mid = (lo_i + hi_i) >> 1;
      if (__ldcg(item_off + mid) <= item) lo_i = mid; else hi_i = mid;
    }
    const int i = lo_i;
    const int g = __ldcg(ws.gemv_list + i);
    const Group gr = ws.groups[g];
    const int units_i = __ldcg(unit_off + i + 1) - __ldcg(unit_off + i);
    const int splits = (__ldcg(item_off + i + 1) - __ldcg(item_off + i)) / units_i;
    const int local = item - __ldcg(item_off + i);
    const int split = local % splits, pass = local / splits;
    const int tp = pass * MT;
    const int mt = min(MT, gr.m - tp);
    const int cnt = __ldcg(ws.union_cnt + g);
    const int lo = static_cast<int>(static_cast<long long>(split) * cnt / splits);
    const int n = static_cast<int>(static_cast<long long>(split + 1) * cnt / splits) - lo;

    // stage the item's rows and h values (fp32, zero past mt)
    const int* rows = ws.union_rows + static_cast<size_t>(g) * dm.F_max + lo;
    const TW* hcol = ht + gr.slot0 + tp;
    for (int r = threadIdx.x; r < n; r += kThreads) {
      const int j = __ldcg(rows + r);
      srow[r] = j;
      float hv[MT];
      load_h<TW, MT>(hcol + static_cast<size_t>(j) * ld, mt, hv);
#pragma unroll
      for (int t = 0; t < MT; ++t) sh[r * MT + t] = hv[t];
    }
    __syncthreads();

    const bool shared = gr.expert >= dm.E;
    const int F_e = shared ? dm.Fs : dm.F;
    const TW* Wbase = shared ? Wds + static_cast<size_t>(gr.expert - dm.E) * F_e * d
                             : Wd + static_cast<size_t>(gr.expert) * F_e * d;
    float* y = ws.y + static_cast<size_t>(gr.slot0 + tp) * d;
    for (int task = warp; task < n_tasks; task += kWarps) {
      const int slice = task % n_slices, phase = task / n_slices;
      const int col = slice * SW + lane * VEC;
      const TW* W = Wbase + col;
      // this warp's rows: p = phase + n_phase * q, q < nq
      const int nq = n > phase ? (n - phase + n_phase - 1) / n_phase : 0;
      const int nb = (nq + kBatch - 1) / kBatch;
      auto issue = [&](int b) {
        if (b < nb) {
          const uint32_t dst = ring_s + (b % kStages) * (kBatch * 512);
#pragma unroll
          for (int r = 0; r < kBatch; ++r) {
            const int q = b * kBatch + r;
            if (q < nq)
              cp_async16(dst + r * 512, W + static_cast<size_t>(srow[phase + n_phase * q]) * d);
          }
        }
        cp_async_commit();
      };
      float acc[MT][VEC];
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[t][v] = 0.f;
#pragma unroll
      for (int b = 0; b < kStages - 1; ++b) issue(b);
      for (int b = 0; b < nb; ++b) {
        issue(b + kStages - 1);
        cp_async_wait<kStages - 1>();
        const uint8_t* src = ring + (b % kStages) * (kBatch * 512) + lane * 16;
#pragma unroll
        for (int r = 0; r < kBatch; ++r) {
          const int q = b * kBatch + r;
          if (q < nq) {
            const uint4 wv = *reinterpret_cast<const uint4*>(src + r * 512);
            float w[VEC];
            Vec<TW>::unpack(wv, w);
            const float* hq = sh + (phase + n_phase * q) * MT;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              const float h = hq[t];
#pragma unroll
              for (int v = 0; v < VEC; ++v) acc[t][v] = fmaf(h, w[v], acc[t][v]);
            }
          }
        }
      }
      cp_async_wait<0>();
      const bool whole = splits == 1 && n_phase == 1;
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t < mt) {
          float* yt = y + static_cast<size_t>(t) * d + col;
#pragma unroll
          for (int v = 0; v < VEC; v += 4) {
            if (whole)
              *reinterpret_cast<float4*>(yt + v) =
                  make_float4(acc[t][v], acc[t][v + 1], acc[t][v + 2], acc[t][v + 3]);
            else
              red_add_v4(yt + v, acc[t][v], acc[t][v + 1], acc[t][v + 2], acc[t][v + 3]);
          }
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace

size_t down_gemv_smem_bytes(bool bf16) {
  const int mt = bf16 ? kGemvTokens : 8;
  return static_cast<size_t>(kWarps) * kWarpRing + sizeof(int) * kGemvRowsMax +
         sizeof(float) * kGemvRowsMax * mt;
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
  const int grid = n_sms;  // one 16-warp CTA per SM
  if (bf16)
    return launch_k(down_gemv_kernel<__nv_bfloat16, kGemvTokens>, grid, kThreads,
                    down_gemv_smem_bytes(true), st, dm, ws,
                    static_cast<const __nv_bfloat16*>(Wd), static_cast<const __nv_bfloat16*>(Wds));
  return launch_k(down_gemv_kernel<float, 8>, grid, kThreads, down_gemv_smem_bytes(false), st,
                  dm, ws, static_cast<const float*>(Wd), static_cast<const float*>(Wds));
}

}  // namespace moe
