// Fused gate + up grouped GEMM on the 5th-generation tensor cores, with the
// SwiGLU / threshold / compaction epilogue.
//
// The gate projection runs densely because its values decide which neurons
// are active [gist.science EN "Uncovering Intra-expert Activation Sparsity
// for Efficient Mixture-of-Expert Model Execution", Technical Summary >
// Methodology > System Implementation in vLLM > "Gate Projection"]; here the
// up projection rides along in the same pass (same B operand, second
// accumulator) because the score is the full SwiGLU value
// h = SiLU(g) * u. The threshold test |h| > tau is one pass over the
// accumulators with no sort [same list, "Activation Masking"].
//
// Work unit: (expert token group, 128-neuron tile), full K = d_model.
//   D_gate[128 neurons][N tokens] = W_gate[e][tile rows] . X_group^T
//   D_up  [128 neurons][N tokens] = W_up  [e][tile rows] . X_group^T
// Neurons are the MMA's M (=128, TMEM lanes) and the group's tokens its N
// (16..256), so decode batches with a handful of tokens per expert still
// use full 128-row MMAs and stream the weights at HBM speed.
//
// Warp roles (192 threads): warp 0 issues TMA loads (A: two 128x64 weight
// boxes, B: N/16 boxes of 16 activation rows, all 128-byte swizzled) into a
// ring of `stages` shared-memory stages; warp 1 owns TMEM and issues
// tcgen05.mma (one thread) and tcgen05.commit; warps 2-5 drain the
// accumulators (tcgen05.ld), compute h in fp32, test |h| > tau before any
// rounding, warp-ballot the active bits of 32 neurons per token, OR them into
// the group's active-row union, and write masked h (bf16) transposed into
// H^T[neuron][slot]. Persistent CTAs walk units with a static stride.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 192;
constexpr uint32_t kABytes = kNeuronTile * kKBlock * 2;  // 16 KB per weight box
constexpr uint32_t kBRowBox = 16;                         // activation rows per B box

struct UnitInfo {
  Group gr;
  int nt;         // neuron tile
  int shared;     // 0 routed, 1 shared
  int F_e;
  int wrow;       // first weight row in the 2-D [experts*F][d] view
};

__device__ __forceinline__ UnitInfo decode_unit(const GateUpTcParams& p, int u, int n_rg,
                                                int tiles_r, int tiles_s) {
  UnitInfo ui;
  int g;
  if (u < n_rg * tiles_r) {
    g = u / tiles_r;
    ui.nt = u % tiles_r;
    ui.shared = 0;
  } else {
    const int v = u - n_rg * tiles_r;
    g = n_rg + v / tiles_s;
    ui.nt = v % tiles_s;
    ui.shared = 1;
  }
  ui.gr = p.ws.groups[g];  // expert: routed e, or E + s for shared expert s
  ui.F_e = ui.shared ? p.dm.Fs : p.dm.F;
  const int e_local = ui.shared ? ui.gr.expert - p.dm.E : ui.gr.expert;
  ui.wrow = e_local * ui.F_e + ui.nt * kNeuronTile;
  return ui;
}

__device__ __forceinline__ int group_of_unit(int u, int n_rg, int tiles_r, int tiles_s) {
  if (u < n_rg * tiles_r) return u / tiles_r;
  return n_rg + (u - n_rg * tiles_r) / tiles_s;
}

__global__ void __launch_bounds__(kThreads, 1)
    gate_up_tc_kernel(const __grid_constant__ GateUpTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  const int n_max = p.n_max;
  const uint32_t stage_bytes = 2 * kABytes + n_max * 128;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  uint64_t* empty = full + stages;
  uint64_t* tfull = empty + stages;  // [2]
  uint64_t* tempty = tfull + 2;      // [2]
  uint64_t* drain = tempty + 2;      // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // TMEM is taken only once the previous kernel has completed, so a CTA of
  // this kernel never holds TMEM while waiting on another kernel
  grid_dep_wait();
  if (warp == 1) tmem_alloc(tmem_slot, p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_rg = __ldcg(p.ws.meta + kMetaRoutedGroups);
  const int n_g = __ldcg(p.ws.meta + kMetaGroups);
  const int tiles_r = p.dm.F / kNeuronTile;
  const int tiles_s = p.dm.S > 0 ? p.dm.Fs / kNeuronTile : 1;
  const int n_units = n_rg * tiles_r + (n_g - n_rg) * tiles_s;
  const int KB = p.dm.d / kKBlock;
  const uint32_t buf_cols = 2u * n_max;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_wg);
      tma_prefetch_desc(&p.tm_wu);
      tma_prefetch_desc(&p.tm_xperm);
      if (p.dm.S > 0) {
        tma_prefetch_desc(&p.tm_wgs);
        tma_prefetch_desc(&p.tm_wus);
        tma_prefetch_desc(&p.tm_x);
      }
    }
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const UnitInfo ui = decode_unit(p, u, n_rg, tiles_r, tiles_s);
      const int N = (ui.gr.m + 15) & ~15;
      const int nb = N / kBRowBox;
      const CUtensorMap* mg = ui.shared ? &p.tm_wgs : &p.tm_wg;
      const CUtensorMap* mu = ui.shared ? &p.tm_wus : &p.tm_wu;
      const CUtensorMap* mx = ui.shared ? &p.tm_x : &p.tm_xperm;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t s = it % stages;
        const uint32_t ph = (it / stages) & 1u;
        if (!warp_wait(empty + s, ph ^ 1u, abort_flag, p.ws.status)) { ok = false; break; }
        uint8_t* sa = smem + s * stage_bytes;
        if (lane == 0) mbar_arrive_expect_tx(full + s, 2 * kABytes + nb * kBRowBox * 128);
        __syncwarp();
        if (lane == 0) {
          tma_load_2d(sa, mg, full + s, kb * kKBlock, ui.wrow);
          tma_load_2d(sa + kABytes, mu, full + s, kb * kKBlock, ui.wrow);
        }
        if (lane < nb)
          tma_load_2d(sa + 2 * kABytes + lane * kBRowBox * 128, mx, full + s, kb * kKBlock,
                      ui.gr.xrow0 + lane * (int)kBRowBox);
        __syncwarp();
      }
    }
    // make sure no copy of ours is still landing when the CTA exits
    const uint32_t n_tail = it < (uint32_t)stages ? it : (uint32_t)stages;
    if (lane == 0) {
      volatile int never = 0;
      for (uint32_t i = it - n_tail; i < it; ++i)
        mbar_wait(full + (i % stages), (i / stages) & 1u, &never, p.ws.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    uint32_t it = 0, uidx = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++uidx) {
      const UnitInfo ui = decode_unit(p, u, n_rg, tiles_r, tiles_s);
      const int N = (ui.gr.m + 15) & ~15;
      const uint32_t idesc = idesc_bf16_f32(kNeuronTile, N, 0, 0);
      const uint32_t b = uidx % p.nbuf;
      const uint32_t tph = (uidx / p.nbuf) & 1u;
      if (!warp_wait(tempty + b, tph ^ 1u, abort_flag, p.ws.status)) break;
      tc_fence_after();
      const uint32_t d_gate = tmem_base + b * buf_cols;
      const uint32_t d_up = d_gate + n_max;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t s = it % stages;
        const uint32_t ph = (it / stages) & 1u;
        if (!warp_wait(full + s, ph, abort_flag, p.ws.status)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sa = smem_u32(smem + s * stage_bytes);
          const uint64_t ag = smem_desc_sw128(sa, 16, 1024);
          const uint64_t au = smem_desc_sw128(sa + kABytes, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sa + 2 * kABytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kKBlock / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0;
            // +32 bytes along K per 16-element step (descriptor units of 16 B)
            mma_bf16(d_gate, ag + 2 * kk, bd + 2 * kk, idesc, acc);
            mma_bf16(d_up, au + 2 * kk, bd + 2 * kk, idesc, acc);
          }
          mma_commit(empty + s);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) mma_commit(tfull + b);
      __syncwarp();
    }
    // all MMAs of this CTA complete before TMEM is released
    if (lane == 0) {
      mma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never, p.ws.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const int fw = p.dm.fw;
    const size_t ld = static_cast<size_t>(p.dm.slots_total);
    __nv_bfloat16* ht = static_cast<__nv_bfloat16*>(p.ws.ht);
    uint32_t uidx = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++uidx) {
      const UnitInfo ui = decode_unit(p, u, n_rg, tiles_r, tiles_s);
      const int g = group_of_unit(u, n_rg, tiles_r, tiles_s);
      const int m = ui.gr.m;
      const int N = (m + 15) & ~15;
      const uint32_t b = uidx % p.nbuf;
      const uint32_t tph = (uidx / p.nbuf) & 1u;
      if (!warp_wait(tfull + b, tph, abort_flag, p.ws.status)) break;
      tc_fence_after();
      const float tau = ui.shared ? p.tau_shared : p.tau;
      const int j = ui.nt * kNeuronTile + 32 * q + lane;  // neuron of this thread
      const int word = (ui.nt * kNeuronTile + 32 * q) >> 5;
      __nv_bfloat16* row = ht + static_cast<size_t>(j) * ld + ui.gr.slot0;
      const uint32_t tg = tmem_base + lane_off + b * buf_cols;
      const uint32_t tu = tg + n_max;
      uint32_t uni = 0;
      unsigned long long nact = 0;
      for (int c0 = 0; c0 < N; c0 += 16) {
        uint32_t gr[16], ur[16];
        tmem_ld16(tg + c0, gr);
        tmem_ld16(tu + c0, ur);
        tmem_ld_wait(gr, ur);
        float hv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = c0 + i;
          const float h = silu_f32(__uint_as_float(gr[i])) * __uint_as_float(ur[i]);
          const bool act = p.dense || fabsf(h) > tau;
          hv[i] = act ? h : 0.f;
          const uint32_t mask = __ballot_sync(0xffffffffu, act && c < m);
          uni |= mask;
          if (lane == 0 && c < m) {
            nact += __popc(mask);
            if (p.ws.act_bits)
              p.ws.act_bits[static_cast<size_t>(ui.gr.slot0 + c) * fw + word] = mask;
          }
        }
        if (c0 + 16 <= m) {
          uint4 pk[2];
          uint32_t* w32 = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            __nv_bfloat162 v2 = __floats2bfloat162_rn(hv[2 * i], hv[2 * i + 1]);
            w32[i] = *reinterpret_cast<uint32_t*>(&v2);
          }
          uint4* dst = reinterpret_cast<uint4*>(row + c0);
          dst[0] = pk[0];
          dst[1] = pk[1];
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < m) row[c0 + i] = __float2bfloat16_rn(hv[i]);
        }
      }
      if (lane == 0) {
        p.ws.union_bits[static_cast<size_t>(g) * fw + word] = uni;
        if (uni) atomicAdd(p.ws.union_cnt + g, __popc(uni));
        atomicAdd(p.ws.counters + (ui.shared ? kCntSharedActive : kCntRoutedActive), nact);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + b);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace

size_t gate_up_tc_smem_bytes(int n_max, int stages) {
  const size_t stage_bytes = 2 * kABytes + static_cast<size_t>(n_max) * 128;
  return 1024 + stages * stage_bytes + (2 * stages + 5) * sizeof(uint64_t) + 16;
}

cudaError_t launch_gate_up_tc(const GateUpTcParams& p, int grid, size_t smem, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gate_up_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_k(gate_up_tc_kernel, grid, kThreads, smem, st, p);
}

}  // namespace moe
