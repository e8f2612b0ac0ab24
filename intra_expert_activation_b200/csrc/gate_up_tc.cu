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
// With the gate score (dm.score_gate) a neuron is active iff |SiLU(g)| > tau
// [same list, "Gate Projection" and "Activation Masking"]; units of groups
// on the GEMV path then load and multiply W_gate only and store the masked
// SiLU(g) in H^T, and the sparse up kernel forms h for the active rows.
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
//
// Whole units leave the SMs unevenly loaded when the unit count is not a
// multiple of the grid (decode: a few experts x d_ff/128 tiles over 148 or
// 296 CTAs, e.g. 896 units = 6 x 148 + 8). So after the rounds of whole
// units, the leftover units are cut along K into at most four parts each and
// spread over the CTAs. A cut unit is finished by the CTA that holds its last
// K-block; the other parts' accumulators go to a per-CTA partial slot with a
// release flag. The finishing CTA meets that unit first in its leftover
// range, parks its own part, and sums the parts and runs the epilogue for it
// after all its other work, when the parts are (nearly) done. Waits are
// bounded; the parts are added in K order. (Cutting every unit's range
// evenly instead lowered the DRAM throughput on small-d layers: the whole-
// unit rounds keep the CTAs in step along K.)
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
  int gate_only;  // gate score and a GEMV group: the up projection is left to the sparse kernel
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
  ui.gate_only = p.dm.sparse_up && __ldcg(p.ws.group_path + g) == kPathGemv;
  ui.F_e = ui.shared ? p.dm.Fs : p.dm.F;
  const int e_local = ui.shared ? ui.gr.expert - p.dm.E : ui.gr.expert;
  ui.wrow = e_local * ui.F_e + ui.nt * kNeuronTile;
  return ui;
}

__device__ __forceinline__ int group_of_unit(int u, int n_rg, int tiles_r, int tiles_s) {
  if (u < n_rg * tiles_r) return u / tiles_r;
  return n_rg + (u - n_rg * tiles_r) / tiles_s;
}

// The CTA's sequence of segments: (unit, first K-block, end K-block). Whole
// units in rounds of G (CTA c takes units c, c + G, ...) while every CTA has
// one; the n_units mod G leftover units are then cut along K, each into at
// most kMaxParts parts, over the first P = min(G, leftover x kMaxParts) CTAs:
// CTA c < P takes iterations [base + Wr c / P, base + Wr (c+1) / P) of the
// Wr = leftover x K-blocks iterations that start at base.
constexpr int kMaxParts = 4;

struct Segs {
  int u, n_full, KB;   // whole units: next one, and how many are whole
  long long i, end;    // leftover iterations of this CTA
};

__device__ __forceinline__ Segs segs_begin(int n_units, int KB, int split) {
  Segs s;
  s.KB = KB;
  s.u = blockIdx.x;
  s.n_full = split ? n_units / gridDim.x * gridDim.x : n_units;
  const int left = n_units - s.n_full;
  const int P = min((int)gridDim.x, left * kMaxParts);
  s.i = s.end = 0;
  if ((int)blockIdx.x < P) {
    const long long base = (long long)s.n_full * KB, Wr = (long long)left * KB;
    s.i = base + Wr * blockIdx.x / P;
    s.end = base + Wr * (blockIdx.x + 1) / P;
  }
  return s;
}

__device__ __forceinline__ bool segs_next(Segs& s, int& u, int& kb0, int& kb1) {
  if (s.u < s.n_full) {
    u = s.u;
    kb0 = 0;
    kb1 = s.KB;
    s.u += gridDim.x;
    return true;
  }
  if (s.i >= s.end) return false;
  u = (int)(s.i / s.KB);
  kb0 = (int)(s.i % s.KB);
  kb1 = (int)min((long long)s.KB, kb0 + (s.end - s.i));
  s.i += kb1 - kb0;
  return true;
}

// CTA holding leftover iteration i.
__device__ __forceinline__ int cta_of_iter(long long i, int n_units, int KB) {
  const int n_full = n_units / gridDim.x * gridDim.x;
  const int left = n_units - n_full;
  const int P = min((int)gridDim.x, left * kMaxParts);
  const long long base = (long long)n_full * KB, Wr = (long long)left * KB;
  return (int)(((i - base + 1) * P - 1) / Wr);
}

// Partial-slot element of (slot, gate|up, 16-column chunk, neuron row, column):
// a warp's 32 rows of one chunk are 2 KB contiguous.
__device__ __forceinline__ float* part_ptr(const GateUpTcParams& p, int slot, int which,
                                           int chunk, int row) {
  const size_t chunks = p.n_max / 16;
  return p.ws.sk_part + ((((size_t)slot * 2 + which) * chunks + chunk) * kNeuronTile + row) * 16;
}

// SwiGLU, threshold and compaction of 16 columns (tokens c0 .. c0+15) of one
// neuron row: masked h to H^T, warp ballots into the union word and counts.
// The score is |h| or, with the gate score, |SiLU(g)|; a gate-only unit
// (sparse up projection to follow) stores the masked SiLU(g) in place of h.
__device__ __forceinline__ void epi_chunk(const GateUpTcParams& p, const UnitInfo& ui, int word,
                                          int c0, int m, float tau, const float (&gv)[16],
                                          const float (&uv)[16], __nv_bfloat16* row,
                                          uint32_t& uni, unsigned long long& nact, int lane) {
  const int fw = p.dm.fw;
  float hv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = c0 + i;
    const float sg = silu_f32(gv[i]);
    const float h = ui.gate_only ? sg : sg * uv[i];
    const bool act = p.dense || fabsf(p.dm.score_gate ? sg : h) > tau;
    hv[i] = act ? h : 0.f;
    const uint32_t mask = __ballot_sync(0xffffffffu, act && c < m);
    uni |= mask;
    if (lane == 0 && c < m) {
      nact += __popc(mask);
      if (p.ws.act_bits) p.ws.act_bits[static_cast<size_t>(ui.gr.slot0 + c) * fw + word] = mask;
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

// Lane 0 of each epilogue warp: the union word, its row count and the
// active-neuron counter of a finished unit.
__device__ __forceinline__ void epi_finish(const GateUpTcParams& p, const UnitInfo& ui, int g,
                                           int word, uint32_t uni, unsigned long long nact,
                                           int lane) {
  if (lane == 0) {
    p.ws.union_bits[static_cast<size_t>(g) * p.dm.fw + word] = uni;
    if (uni) atomicAdd(p.ws.union_cnt + g, __popc(uni));
    atomicAdd(p.ws.counters + (ui.shared ? kCntSharedActive : kCntRoutedActive), nact);
  }
}

// The four epilogue warps only (named barrier 1).
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    gate_up_tc_kernel(const __grid_constant__ GateUpTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  const int n_max = p.n_max;
  // stage: two 16 KB weight boxes, then b_blocks activation regions of n_max
  // rows (with the gate score a gate-only unit puts two K-blocks of W_gate and
  // of x in one stage, so that a stage still carries two weight boxes)
  const uint32_t b_half = n_max * 128;
  const uint32_t stage_bytes = 2 * kABytes + p.b_blocks * b_half;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  uint64_t* empty = full + stages;
  uint64_t* tfull = empty + stages;  // [2]
  uint64_t* tempty = tfull + 2;      // [2]
  uint64_t* drain = tempty + 2;      // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* fix_ok = abort_flag + 1;  // the parked unit's parts are all published

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
  const int split = p.split;

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
    Segs sg = segs_begin(n_units, KB, split);
    int u, kb0, kb1;
    while (ok && segs_next(sg, u, kb0, kb1)) {
      const UnitInfo ui = decode_unit(p, u, n_rg, tiles_r, tiles_s);
      const int N = (ui.gr.m + 15) & ~15;
      const int nb = N / kBRowBox;
      const CUtensorMap* mg = ui.shared ? &p.tm_wgs : &p.tm_wg;
      const CUtensorMap* mu = ui.shared ? &p.tm_wus : &p.tm_wu;
      const CUtensorMap* mx = ui.shared ? &p.tm_x : &p.tm_xperm;
      const int kstep = ui.gate_only && p.b_blocks == 2 ? 2 : 1;  // K-blocks per stage
      for (int kb = kb0; kb < kb1; kb += kstep, ++it) {
        const uint32_t s = it % stages;
        const uint32_t ph = (it / stages) & 1u;
        if (!warp_wait(empty + s, ph ^ 1u, abort_flag, p.ws.status)) { ok = false; break; }
        uint8_t* sa = smem + s * stage_bytes;
        const int nk = min(kstep, kb1 - kb);
        const uint32_t xbytes = nb * kBRowBox * 128;
        if (lane == 0)
          mbar_arrive_expect_tx(full + s, ui.gate_only ? nk * (kABytes + xbytes)
                                                       : 2 * kABytes + xbytes);
        __syncwarp();
        if (ui.gate_only) {  // W_gate and x of K-blocks kb (, kb + 1)
          for (int j = 0; j < nk; ++j) {
            if (lane == 0) tma_load_2d(sa + j * kABytes, mg, full + s, (kb + j) * kKBlock, ui.wrow);
            if (lane < nb)
              tma_load_2d(sa + 2 * kABytes + j * b_half + lane * kBRowBox * 128, mx, full + s,
                          (kb + j) * kKBlock, ui.gr.xrow0 + lane * (int)kBRowBox);
          }
        } else {
          if (lane == 0) {
            tma_load_2d(sa, mg, full + s, kb * kKBlock, ui.wrow);
            tma_load_2d(sa + kABytes, mu, full + s, kb * kKBlock, ui.wrow);
          }
          if (lane < nb)
            tma_load_2d(sa + 2 * kABytes + lane * kBRowBox * 128, mx, full + s, kb * kKBlock,
                        ui.gr.xrow0 + lane * (int)kBRowBox);
        }
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
    Segs sg = segs_begin(n_units, KB, split);
    int u, kb0, kb1;
    for (; ok && segs_next(sg, u, kb0, kb1); ++uidx) {
      const UnitInfo ui = decode_unit(p, u, n_rg, tiles_r, tiles_s);
      const int N = (ui.gr.m + 15) & ~15;
      const uint32_t idesc = idesc_bf16_f32(kNeuronTile, N, 0, 0);
      const uint32_t b = uidx % p.nbuf;
      const uint32_t tph = (uidx / p.nbuf) & 1u;
      if (!warp_wait(tempty + b, tph ^ 1u, abort_flag, p.ws.status)) break;
      tc_fence_after();
      const uint32_t d_gate = tmem_base + b * buf_cols;
      const uint32_t d_up = d_gate + n_max;
      const int kstep = ui.gate_only && p.b_blocks == 2 ? 2 : 1;  // K-blocks per stage
      for (int kb = kb0; kb < kb1; kb += kstep, ++it) {
        const uint32_t s = it % stages;
        const uint32_t ph = (it / stages) & 1u;
        if (!warp_wait(full + s, ph, abort_flag, p.ws.status)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sa = smem_u32(smem + s * stage_bytes);
          if (ui.gate_only) {
            const int nk = min(kstep, kb1 - kb);
            for (int j = 0; j < nk; ++j) {
              const uint64_t ag = smem_desc_sw128(sa + j * kABytes, 16, 1024);
              const uint64_t bd = smem_desc_sw128(sa + 2 * kABytes + j * b_half, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < kKBlock / 16; ++kk)
                mma_bf16(d_gate, ag + 2 * kk, bd + 2 * kk, idesc, (kb + j != kb0) || (kk != 0));
            }
          } else {
            const uint64_t ag = smem_desc_sw128(sa, 16, 1024);
            const uint64_t au = smem_desc_sw128(sa + kABytes, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sa + 2 * kABytes, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < kKBlock / 16; ++kk) {
              const uint32_t acc = (kb != kb0) || (kk != 0);
              // +32 bytes along K per 16-element step (descriptor units of 16 B)
              mma_bf16(d_gate, ag + 2 * kk, bd + 2 * kk, idesc, acc);
              mma_bf16(d_up, au + 2 * kk, bd + 2 * kk, idesc, acc);
            }
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
    const size_t ld = static_cast<size_t>(p.dm.slots_total);
    __nv_bfloat16* ht = static_cast<__nv_bfloat16*>(p.ws.ht);
    uint32_t uidx = 0;
    bool ok = true;
    int park_u = -1;  // split unit whose last K-block is ours: finished at the end
    Segs sg = segs_begin(n_units, KB, split);
    int u, kb0, kb1;
    for (; segs_next(sg, u, kb0, kb1); ++uidx) {
      // every epilogue warp walks every segment (named barriers below), doing
      // nothing once a wait has failed
      const UnitInfo ui = decode_unit(p, u, n_rg, tiles_r, tiles_s);
      const int g = group_of_unit(u, n_rg, tiles_r, tiles_s);
      const int m = ui.gr.m;
      const int N = (m + 15) & ~15;
      const uint32_t b = uidx % p.nbuf;
      const uint32_t tph = (uidx / p.nbuf) & 1u;
      if (ok && !warp_wait(tfull + b, tph, abort_flag, p.ws.status)) ok = false;
      const bool whole = kb0 == 0 && kb1 == KB;
      const bool last_part = !whole && kb1 == KB;
      if (ok) {
        tc_fence_after();
        const float tau = ui.shared ? p.tau_shared : p.tau;
        const int row_i = 32 * q + lane;
        const int j = ui.nt * kNeuronTile + row_i;  // neuron of this thread
        const int word = (ui.nt * kNeuronTile + 32 * q) >> 5;
        __nv_bfloat16* row = ht + static_cast<size_t>(j) * ld + ui.gr.slot0;
        const uint32_t tg = tmem_base + lane_off + b * buf_cols;
        const uint32_t tu = tg + n_max;
        uint32_t uni = 0;
        unsigned long long nact = 0;
        const int slot = last_part ? gridDim.x + blockIdx.x : blockIdx.x;
        for (int c0 = 0; c0 < N; c0 += 16) {
          uint32_t gr[16], ur[16];
          tmem_ld16(tg + c0, gr);
          if (ui.gate_only) {
            tmem_ld_wait(gr);
#pragma unroll
            for (int i = 0; i < 16; ++i) ur[i] = 0u;
          } else {
            tmem_ld16(tu + c0, ur);
            tmem_ld_wait(gr, ur);
          }
          float gv[16], uv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            gv[i] = __uint_as_float(gr[i]);
            uv[i] = __uint_as_float(ur[i]);
          }
          if (whole) {
            epi_chunk(p, ui, word, c0, m, tau, gv, uv, row, uni, nact, lane);
          } else {  // a part of a split unit: park its sums
            float4* pg = reinterpret_cast<float4*>(part_ptr(p, slot, 0, c0 / 16, row_i));
            float4* pu = reinterpret_cast<float4*>(part_ptr(p, slot, 1, c0 / 16, row_i));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              pg[i] = make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]);
              pu[i] = make_float4(uv[4 * i], uv[4 * i + 1], uv[4 * i + 2], uv[4 * i + 3]);
            }
          }
        }
        if (whole) {
          epi_finish(p, ui, g, word, uni, nact, lane);
          if (q == 0 && lane == 0)  // weight rows this unit loaded
            atomicAdd(p.ws.counters + kCntGateUpRows, (ui.gate_only ? 1ull : 2ull) * kNeuronTile);
        }
      }
      if (last_part) park_u = u;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + b);
      if (!whole && !last_part) {
        // an earlier part: publish it for the CTA that holds the unit's end
        __threadfence();
        epi_sync();
        if (warp == 2 && lane == 0)
          asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p.ws.sk_flags + blockIdx.x),
                       "r"(1)
                       : "memory");
      }
    }
    if (park_u >= 0) {
      // sum the parts of the parked unit in K order, then its epilogue
      const int c_first = cta_of_iter((long long)park_u * KB, n_units, KB);
      if (warp == 2 && lane == 0) {
        int good = *abort_flag == 0 ? 1 : 0;
        for (int c2 = c_first; c2 < (int)blockIdx.x && good; ++c2)
          good = wait_flag(p.ws.sk_flags + c2, abort_flag, p.ws.status) ? 1 : 0;
        *fix_ok = good;
      }
      epi_sync();
      if (*fix_ok) {
        const UnitInfo ui = decode_unit(p, park_u, n_rg, tiles_r, tiles_s);
        const int g = group_of_unit(park_u, n_rg, tiles_r, tiles_s);
        const int m = ui.gr.m;
        const int N = (m + 15) & ~15;
        const float tau = ui.shared ? p.tau_shared : p.tau;
        const int row_i = 32 * q + lane;
        const int j = ui.nt * kNeuronTile + row_i;
        const int word = (ui.nt * kNeuronTile + 32 * q) >> 5;
        __nv_bfloat16* row = ht + static_cast<size_t>(j) * ld + ui.gr.slot0;
        uint32_t uni = 0;
        unsigned long long nact = 0;
        for (int c0 = 0; c0 < N; c0 += 16) {
          float gv[16], uv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) gv[i] = uv[i] = 0.f;
          for (int c2 = c_first; c2 <= (int)blockIdx.x; ++c2) {
            const int slot = c2 == (int)blockIdx.x ? gridDim.x + blockIdx.x : c2;
            const float4* pg = reinterpret_cast<const float4*>(part_ptr(p, slot, 0, c0 / 16, row_i));
            const float4* pu = reinterpret_cast<const float4*>(part_ptr(p, slot, 1, c0 / 16, row_i));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float4 a = __ldcg(pg + i), c = __ldcg(pu + i);
              gv[4 * i] += a.x; gv[4 * i + 1] += a.y; gv[4 * i + 2] += a.z; gv[4 * i + 3] += a.w;
              uv[4 * i] += c.x; uv[4 * i + 1] += c.y; uv[4 * i + 2] += c.z; uv[4 * i + 3] += c.w;
            }
          }
          epi_chunk(p, ui, word, c0, m, tau, gv, uv, row, uni, nact, lane);
        }
        epi_finish(p, ui, g, word, uni, nact, lane);
        if (q == 0 && lane == 0)
          atomicAdd(p.ws.counters + kCntGateUpRows, (ui.gate_only ? 1ull : 2ull) * kNeuronTile);
      }
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

size_t gate_up_tc_smem_bytes(int n_max, int stages, int b_blocks) {
  const size_t stage_bytes = 2 * kABytes + static_cast<size_t>(b_blocks) * n_max * 128;
  return 1024 + stages * stage_bytes + (2 * stages + 5) * sizeof(uint64_t) + 16;
}

cudaError_t launch_gate_up_tc(const GateUpTcParams& p, int grid, size_t smem, cudaStream_t st) {
  const cudaError_t e = smem_limit(gate_up_tc_kernel, 227 * 1024);
  if (e != cudaSuccess) return e;
  return launch_k(gate_up_tc_kernel, grid, kThreads, smem, st, p);
}

}  // namespace moe
