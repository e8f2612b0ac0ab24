// fp32 gate + up projections with the SwiGLU / threshold epilogue on CUDA
// cores, for layers stored in fp32 (the tensor cores' tf32 mode would not
// keep the fp32 accuracy). Same outputs as the tensor-core kernel: masked h
// transposed into H^T[neuron][slot] (fp32 here), the group's active-row
// union bitmap and, with debugging on, per-slot active bitmaps. With the
// gate score only the gate projection runs here and H^T receives the masked
// SiLU(g) (the sparse up kernel completes h).
// [gist.science EN "Uncovering Intra-expert Activation Sparsity for Efficient
// Mixture-of-Expert Model Execution", Technical Summary > Methodology >
// System Implementation in vLLM > "Gate Projection" and "Activation Masking"]
//
// Work unit: (group, 32-neuron block) = one bitmap word per token. Each warp
// owns 4 neurons and evaluates their gate and up dot products for every
// token of the group (lanes stride d, butterfly reduction: a fixed order).
#include "common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    gate_up_simt_kernel(Dims dm, Workspace ws, const float* __restrict__ x,
                        const float* __restrict__ Wg, const float* __restrict__ Wu,
                        const float* __restrict__ Wgs, const float* __restrict__ Wus, float tau,
                        float tau_shared, int dense) {
  __shared__ uint32_t tok_bits[kGroupMax];
  __shared__ uint32_t uni;
  grid_dep_wait();
  const int n_rg = __ldcg(ws.meta + kMetaRoutedGroups);
  const int n_g = __ldcg(ws.meta + kMetaGroups);
  const int blk_r = dm.F / 32;
  const int blk_s = dm.S > 0 ? dm.Fs / 32 : 1;
  const int n_units = n_rg * blk_r + (n_g - n_rg) * blk_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = dm.d;
  const size_t ld = static_cast<size_t>(dm.slots_total);
  float* ht = static_cast<float*>(ws.ht);
  const float* xperm = static_cast<const float*>(ws.xperm);

  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    int g, blk;
    if (u < n_rg * blk_r) {
      g = u / blk_r;
      blk = u % blk_r;
    } else {
      g = n_rg + (u - n_rg * blk_r) / blk_s;
      blk = (u - n_rg * blk_r) % blk_s;
    }
    const Group gr = ws.groups[g];
    const bool shared = gr.expert >= dm.E;
    const int F_e = shared ? dm.Fs : dm.F;
    const float* Wge = shared ? Wgs + static_cast<size_t>(gr.expert - dm.E) * F_e * d
                              : Wg + static_cast<size_t>(gr.expert) * F_e * d;
    const float* Wue = shared ? Wus + static_cast<size_t>(gr.expert - dm.E) * F_e * d
                              : Wu + static_cast<size_t>(gr.expert) * F_e * d;
    const float* X = shared ? x : xperm;
    const float th = shared ? tau_shared : tau;
    const bool gate_only = dm.sparse_up != 0;

    for (int t = threadIdx.x; t < gr.m; t += kThreads) tok_bits[t] = 0u;
    if (threadIdx.x == 0) uni = 0u;
    __syncthreads();

    for (int jj = 0; jj < 4; ++jj) {
      const int j = blk * 32 + warp * 4 + jj;
      const float* wg = Wge + static_cast<size_t>(j) * d;
      const float* wu = Wue + static_cast<size_t>(j) * d;
      for (int t = 0; t < gr.m; ++t) {
        const float* xr = X + static_cast<size_t>(gr.xrow0 + t) * d;
        float gs = 0.f, us = 0.f;
        for (int i = lane; i < d; i += 32) {
          const float xv = xr[i];
          gs = fmaf(xv, wg[i], gs);
          if (!gate_only) us = fmaf(xv, wu[i], us);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          gs += __shfl_xor_sync(0xffffffffu, gs, o);
          us += __shfl_xor_sync(0xffffffffu, us, o);
        }
        // gate score: active iff |SiLU(g)| > tau; with the sparse up
        // projection the masked SiLU(g) is stored for the fused up + down
        // kernel (every fp32 group is on the GEMV path), else the masked h
        const float sg = silu_f32(gs);
        const float h = gate_only ? sg : sg * us;
        const bool act = dense || fabsf(dm.score_gate ? sg : h) > th;
        if (lane == 0) {
          ht[static_cast<size_t>(j) * ld + gr.slot0 + t] = act ? h : 0.f;
          if (act) atomicOr(&tok_bits[t], 1u << (j & 31));
        }
      }
    }
    __syncthreads();
    unsigned long long nact = 0;
    for (int t = threadIdx.x; t < gr.m; t += kThreads) {
      const uint32_t w = tok_bits[t];
      if (ws.act_bits) ws.act_bits[static_cast<size_t>(gr.slot0 + t) * dm.fw + blk] = w;
      atomicOr(&uni, w);
      nact += __popc(w);
    }
    if (nact) atomicAdd(ws.counters + (shared ? kCntSharedActive : kCntRoutedActive), nact);
    __syncthreads();
    if (threadIdx.x == 0) {
      ws.union_bits[static_cast<size_t>(g) * dm.fw + blk] = uni;
      if (uni) atomicAdd(ws.union_cnt + g, __popc(uni));
      atomicAdd(ws.counters + kCntGateUpRows, (gate_only ? 1ull : 2ull) * 32ull);
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_gate_up_simt(const Dims& dm, const Workspace& ws, const float* x,
                                const float* Wg, const float* Wu, const float* Wgs,
                                const float* Wus, float tau, float tau_shared, int dense,
                                cudaStream_t st) {
  const int units_max = dm.groups_max * (dm.F_max / 32);
  const int grid = units_max < 4096 ? units_max : 4096;
  return launch_k(gate_up_simt_kernel, grid, kThreads, 0, st, dm, ws, x, Wg, Wu, Wgs, Wus, tau,
                  tau_shared, dense);
}

}  // namespace moe
