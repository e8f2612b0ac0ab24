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
//
// Fused down projection (groups of kPathFused: the smallest row-stream
// groups of batches whose units fit one per CTA, dm.fuse_down). Once a
// unit's h is known, the tile's active rows are final: neuron j of the tile
// contributes h_j W_down[e][j,:] to the group's outputs and nothing else does
// [same list, "Fused Up-Down Projection": only the active neurons' weight
// rows are fetched]. So after the unit's epilogue (its TMEM buffer handed
// back to the MMA warp) the four epilogue warps compact the tile's active
// rows and their h values into shared memory; as the CTA's last work, when
// its weight ring is idle, they bring those rows of W_down into the ring by
// bulk copies, multiply on the CUDA cores in fp32 and add the sums into Y
// with vector fp32 atomics (or, under direct combine, w x the sums into the
// token's output accumulator row, the last CTA writing out). A unit that is
// not its CTA's last (not the case the host arranges) reads the rows with
// 16-byte loads instead. This saves the row-stream kernel's launch, start-up
// and walk over the union bitmaps. h is rounded to bf16 first, as H^T holds
// it for the down kernels. With the gate score a one-token group's unit is
// gate-only: its active rows (|SiLU(g)| > tau) of W_up come through the ring
// first, dotted with the token's x, and then the same rows of W_down.
#include "common.cuh"
#include "topk.cuh"

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
  int fused;      // kPathFused: this kernel also does the unit's down projection
};

// One-token routing inside this kernel (dm.route1): the selected experts in
// expert order (group g = the g-th of them, its slot block g) and their
// combine weights.
struct Route1Groups {
  int k;
  int exp[16];
  float w[16];
};

__device__ __forceinline__ UnitInfo decode_unit(const GateUpTcParams& p, int u, int n_rg,
                                                int tiles_r, int tiles_s,
                                                const Route1Groups* r1) {
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
  int path;
  if (r1) {  // the token (row 0 of x) alone, in slot block g
    ui.gr.expert = r1->exp[g];
    ui.gr.slot0 = g * kSlotAlign;
    ui.gr.m = 1;
    ui.gr.xrow0 = 0;
    path = kPathFused;
  } else {
    ui.gr = p.ws.groups[g];  // expert: routed e, or E + s for shared expert s
    path = __ldcg(p.ws.group_path + g);
  }
  ui.gate_only = p.dm.sparse_up && (path == kPathGemv || path == kPathFused);
  ui.fused = path == kPathFused;
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
// Wr = leftover x K-blocks iterations that start at base. Only a short last
// round is cut (fewer leftover units than half the grid): a last round that
// fills most of the grid runs as whole units (measured on the Mixtral-shaped
// layer: cutting 192 leftover units of 296 slots cost 7 us at T = 8, cutting
// 8 leftover units saved 15-20 us at T = 32 and 64).
constexpr int kMaxParts = 4;

__device__ __forceinline__ int whole_units(int n_units, int split) {
  const int G = gridDim.x;
  return split && 2 * (n_units % G) < G ? n_units / G * G : n_units;
}

struct Segs {
  int u, n_full, KB;   // whole units: next one, and how many are whole
  long long i, end;    // leftover iterations of this CTA
};

__device__ __forceinline__ Segs segs_begin(int n_units, int KB, int split) {
  Segs s;
  s.KB = KB;
  s.u = blockIdx.x;
  s.n_full = whole_units(n_units, split);
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
  const int n_full = whole_units(n_units, 1);  // only called for cut units
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
// hv receives the masked values (columns past m hold values of padding rows).
__device__ __forceinline__ void epi_chunk(const GateUpTcParams& p, const UnitInfo& ui, int word,
                                          int c0, int m, float tau, const float (&gv)[16],
                                          const float (&uv)[16], __nv_bfloat16* row,
                                          uint32_t& uni, unsigned long long& nact, int lane,
                                          float (&hv)[16]) {
  const int fw = p.dm.fw;
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

// ------------------------------------------------------------ fused down projection

// Shared-memory scratch of one unit's fused down projection: the tile's
// active rows in neuron order with their h values (bf16-rounded, zero for
// the tokens where the row is inactive).
constexpr int kFuseHalfMax = 32;  // rows per half of the ring in the bulk path

struct FuseScratch {
  uint64_t bar[2];            // bulk-copy halves of the ring (last unit of a CTA)
  alignas(16) float h[kNeuronTile][kFuseTokens];  // read as float4 rows
  uint8_t rows[kNeuronTile];  // neuron index within the tile
  int cnt[4];                 // active rows of each epilogue warp's 32 neurons
  float red[4][kFuseHalfMax]; // gate score: the four warps' partial up dots of a batch
  Route1Groups r1;            // dm.route1: this CTA's routing of the token
};
static_assert(offsetof(FuseScratch, h) % 16 == 0, "h rows are read as float4");
constexpr int kFuseCols = 8;      // bf16 columns per thread and load (16 bytes)
constexpr int kFuseInFlight = 16;  // row loads in flight per thread

// Epilogue warps: place this warp's active neurons (bits of uni; hv their h
// values, token t in hv[t]) at their rank among the tile's active rows.
// Returns the tile's active row count. Every epilogue warp calls it.
__device__ __forceinline__ int fuse_compact(FuseScratch& fs, uint32_t uni,
                                            const float (&hv)[kFuseTokens], int m, int q,
                                            int lane) {
  if (lane == 0) fs.cnt[q] = __popc(uni);
  epi_sync();
  int off = 0, R = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int c = fs.cnt[w];
    off += w < q ? c : 0;
    R += c;
  }
  if ((uni >> lane) & 1u) {
    const int pos = off + __popc(uni & ((1u << lane) - 1u));
    fs.rows[pos] = static_cast<uint8_t>(32 * q + lane);
#pragma unroll
    for (int t = 0; t < kFuseTokens; ++t)
      fs.h[pos][t] = t < m ? __bfloat162float(__float2bfloat16_rn(hv[t])) : 0.f;
  }
  epi_sync();
  return R;
}

// acc[t][8 k + i] += h[t] * w[i] for the 8 bf16 values w of v.
template <int MT, int KC>
__device__ __forceinline__ void fuse_fma(float (&acc)[MT][KC * kFuseCols], int k, const uint4& v,
                                         const float* h) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  float w[kFuseCols];
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // bf16 -> fp32: the high half of a 32-bit word
    w[2 * i] = __uint_as_float(u[i] << 16);
    w[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
  float hh[MT];
  if constexpr (MT == 4) {
    const float4 h4 = *reinterpret_cast<const float4*>(h);
    hh[0] = h4.x; hh[1] = h4.y; hh[2] = h4.z; hh[3] = h4.w;
  } else {
#pragma unroll
    for (int t = 0; t < MT; ++t) hh[t] = h[t];
  }
#pragma unroll
  for (int t = 0; t < MT; ++t)
#pragma unroll
    for (int i = 0; i < kFuseCols; ++i)
      acc[t][k * kFuseCols + i] = fmaf(hh[t], w[i], acc[t][k * kFuseCols + i]);
}

// The unit's down projection over its R compacted rows, by the 128 epilogue
// threads (tid 0..127). Thread tid owns columns 8 tid + 1024 k + [0, 8) for
// k < KC of every 1024 KC-column block of d and the group's MT token slots
// (m <= MT). Each batch issues kFuseInFlight 16-byte loads (kFuseInFlight /
// KC rows, KC pieces of 2 KB of each) before using the first: with KC = 4 the
// 128 threads request whole 8 KB rows (d = 4096) at once, which streams
// faster than 2 KB pieces of many rows; the accumulators (MT x KC x 8) stay
// at 32 registers.
template <int MT, int KC>
__device__ void fuse_cols(const GateUpTcParams& p, const UnitInfo& ui, const FuseScratch& fs,
                          int R, int tid) {
  constexpr int RB = kFuseInFlight / KC;  // rows per batch
  const int d = p.dm.d, m = ui.gr.m;
  const __nv_bfloat16* W = (ui.shared ? p.wds : p.wd) + static_cast<size_t>(ui.wrow) * d;
  float* yrow[MT];
  float wt[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    yrow[t] = nullptr;
    wt[t] = 1.f;
    if (t < m) {
      int tok = ui.gr.slot0 + t;
      if (p.dm.direct_combine) slot_target(p.dm, p.ws, ui.gr.slot0 + t, tok, wt[t]);
      yrow[t] = p.ws.y + static_cast<size_t>(tok) * d;
    }
  }
  for (int c0 = tid * kFuseCols; c0 < d; c0 += 128 * kFuseCols * KC) {
    float acc[MT][KC * kFuseCols];
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int i = 0; i < KC * kFuseCols; ++i) acc[t][i] = 0.f;
    const __nv_bfloat16* wc = W + c0;
    for (int r = 0; r < R; r += RB) {
      // all loads of the batch are issued before the first is used (rows past
      // R re-read the last row, which is not multiplied)
      uint4 v[RB][KC];
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        const int rr = min(r + u, R - 1);
        const __nv_bfloat16* wr = wc + static_cast<size_t>(fs.rows[rr]) * d;
#pragma unroll
        for (int k = 0; k < KC; ++k) v[u][k] = ld_stream_v4(wr + k * 128 * kFuseCols);
      }
#pragma unroll
      for (int u = 0; u < RB; ++u)
        if (r + u < R)
#pragma unroll
          for (int k = 0; k < KC; ++k) fuse_fma<MT, KC>(acc, k, v[u][k], fs.h[r + u]);
    }
#pragma unroll
    for (int t = 0; t < MT; ++t)
      if (t < m) {
        const float w = wt[t];
#pragma unroll
        for (int k = 0; k < KC; ++k) {
          float* y = yrow[t] + c0 + k * 128 * kFuseCols;
          const float* a = acc[t] + k * kFuseCols;
          red_add_v4(y, w * a[0], w * a[1], w * a[2], w * a[3]);
          red_add_v4(y + 4, w * a[4], w * a[5], w * a[6], w * a[7]);
        }
      }
  }
}

// The CTA's last unit (its weight ring is idle: every copy landed and every
// MMA that read the ring has completed): the unit's R compacted rows of a
// matrix W (W_down, or with the gate score first W_up), whole (d = 1024 KC,
// rows of 2 KB KC), come into the ring by bulk copies, H rows per half, the
// two halves alternating, so that up to 2 H rows are in flight while the 128
// threads use the landed half from shared memory (thread tid reads 16 bytes
// at 2 KB k + 16 tid of a row: conflict-free). row(r, i, src) is called by
// every thread for landed row r (i-th of its batch, src: the thread's first
// 16 bytes of it), batch(r0, n) by every thread after each batch (it may use
// epi_sync), then the half is freed. fz_it counts the batches on the two
// half barriers, whose phases run on from one call to the next. Returns
// false once a wait has failed (the copies in flight have landed then).
template <class RowFn, class BatchFn>
__device__ bool bulk_rows(const GateUpTcParams& p, FuseScratch& fs, const __nv_bfloat16* W,
                          int R, int tid, uint8_t* ring, uint32_t ring_bytes, uint32_t& fz_it,
                          volatile int* abort_flag, RowFn row, BatchFn batch) {
  const int d = p.dm.d;
  const uint32_t row_bytes = static_cast<uint32_t>(d) * 2;
  const int H = min(static_cast<int>(ring_bytes / row_bytes) / 2, kFuseHalfMax);
  const int nb = (R + H - 1) / H;
  const uint32_t g0 = fz_it;  // barrier index of this call's batch 0
  fz_it += static_cast<uint32_t>(nb);
  auto issue = [&](int b) {  // thread 0: batch b into half (g0 + b) & 1
    const int h = (g0 + b) & 1, r0 = b * H, n = min(H, R - r0);
    mbar_arrive_expect_tx(&fs.bar[h], static_cast<uint32_t>(n) * row_bytes);
    for (int i = 0; i < n; ++i)
      bulk_load(smem_u32(ring + static_cast<size_t>(h * H + i) * row_bytes),
                W + static_cast<size_t>(fs.rows[r0 + i]) * d, row_bytes, smem_u32(&fs.bar[h]));
  };
  int issued = 0;  // thread 0: batches issued
  if (tid == 0) {
    issue(0);
    issued = 1;
    if (nb > 1) {
      issue(1);
      issued = 2;
    }
  }
  bool ok = true;
  for (int b = 0; b < nb; ++b) {
    // every epilogue warp runs every batch (named barriers), skipping the
    // work once a wait has failed
    const uint32_t g = g0 + b;
    const int h = g & 1;
    if (ok && !warp_wait(&fs.bar[h], (g >> 1) & 1, abort_flag, p.ws.status)) ok = false;
    const int r0 = b * H, n = min(H, R - r0);
    if (ok) {
      const uint8_t* base = ring + static_cast<size_t>(h * H) * row_bytes + tid * 16;
      for (int i = 0; i < n; ++i) row(r0 + i, i, base + static_cast<size_t>(i) * row_bytes);
    }
    batch(r0, n);
    epi_sync();  // the half is read: it may be refilled
    if (tid == 0 && b + 2 < nb && !*abort_flag) {
      issue(b + 2);
      issued = b + 3;
    }
  }
  if (tid == 0 && *abort_flag) {
    // copies still in flight land before the CTA may exit: wait (bounded) for
    // the last batch issued on each half
    volatile int never = 0;
    for (int hh = 0; hh < 2; ++hh) {
      int lb = issued - 1;  // this call's last batch on half hh
      if (lb >= 0 && static_cast<int>((g0 + lb) & 1) != hh) --lb;
      if (lb >= 0) mbar_wait(&fs.bar[hh], ((g0 + lb) >> 1) & 1, &never, p.ws.status);
    }
  }
  return ok && !*abort_flag;
}

// Adds w x the sums of this thread's columns (tokens t < m of the group,
// acc[t][8 k + i] at column 8 tid + 1024 k + i) into Y or, under direct
// combine, into the tokens' output accumulator rows.
template <int MT, int KC>
__device__ __forceinline__ void fuse_flush(const GateUpTcParams& p, const UnitInfo& ui,
                                           const float (&acc)[MT][KC * kFuseCols], int m,
                                           int tid) {
  const int d = p.dm.d;
  const int c0 = tid * kFuseCols;
#pragma unroll
  for (int t = 0; t < MT; ++t)
    if (t < m) {
      int tok = ui.gr.slot0 + t;
      float w = 1.f;
      if (p.dm.direct_combine) slot_target(p.dm, p.ws, ui.gr.slot0 + t, tok, w);
      float* yrow = p.ws.y + static_cast<size_t>(tok) * d;
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        float* y = yrow + c0 + k * 128 * kFuseCols;
        const float* a = acc[t] + k * kFuseCols;
        red_add_v4(y, w * a[0], w * a[1], w * a[2], w * a[3]);
        red_add_v4(y + 4, w * a[4], w * a[5], w * a[6], w * a[7]);
      }
    }
}

// The last unit's down projection through the ring: y += h_r W_down[r] over
// its R rows, tokens t < m <= MT (MT <= 2 keeps the accumulators at <= 64
// registers).
template <int MT, int KC>
__device__ void fuse_rows_bulk(const GateUpTcParams& p, const UnitInfo& ui, FuseScratch& fs,
                               int R, int tid, uint8_t* ring, uint32_t ring_bytes,
                               uint32_t& fz_it, volatile int* abort_flag) {
  float acc[MT][KC * kFuseCols];
#pragma unroll
  for (int t = 0; t < MT; ++t)
#pragma unroll
    for (int i = 0; i < KC * kFuseCols; ++i) acc[t][i] = 0.f;
  const __nv_bfloat16* W = (ui.shared ? p.wds : p.wd) + static_cast<size_t>(ui.wrow) * p.dm.d;
  const bool ok = bulk_rows(
      p, fs, W, R, tid, ring, ring_bytes, fz_it, abort_flag,
      [&](int r, int, const uint8_t* src) {
#pragma unroll
        for (int k = 0; k < KC; ++k)
          fuse_fma<MT, KC>(acc, k, *reinterpret_cast<const uint4*>(src + k * 2048), fs.h[r]);
      },
      [&](int, int) {});
  if (ok) fuse_flush<MT, KC>(p, ui, acc, ui.gr.m, tid);
}

// Gate score, a one-token group (the last unit of its CTA): the unit's rows
// are the neurons with |SiLU(g)| > tau, and fs.h holds their SiLU(g) rounded
// to bf16. First the rows of W_up come through the ring: each thread dots
// its columns of a row with the token's x (kept in registers), the four
// warps' partials of a batch meet in shared memory and are added in warp
// order, and h = bf16(SiLU(g) u) replaces SiLU(g) in fs.h (as the separate
// fused kernel rounds it); then the same rows of W_down, as fuse_rows_bulk
// [same list, "Fused Up-Down Projection": only the active neurons' up and
// down weights are fetched].
template <int KC>
__device__ void fuse_updown_bulk(const GateUpTcParams& p, const UnitInfo& ui, FuseScratch& fs,
                                 int R, int tid, uint8_t* ring, uint32_t ring_bytes,
                                 uint32_t& fz_it, volatile int* abort_flag) {
  const int d = p.dm.d;
  const int q = tid >> 5, lane = tid & 31;
  // the token's x: routed groups from X_perm, shared experts' from x
  const __nv_bfloat16* xr =
      (ui.shared || p.dm.route1 ? p.x : static_cast<const __nv_bfloat16*>(p.ws.xperm)) +
      static_cast<size_t>(ui.gr.xrow0) * d;
  float xv[KC * kFuseCols];
#pragma unroll
  for (int k = 0; k < KC; ++k) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr + tid * kFuseCols + k * 1024));
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xv[k * kFuseCols + 2 * i] = __uint_as_float(u[i] << 16);
      xv[k * kFuseCols + 2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
  }
  const __nv_bfloat16* Wu = (ui.shared ? p.wus : p.wu) + static_cast<size_t>(ui.wrow) * d;
  const bool ok = bulk_rows(
      p, fs, Wu, R, tid, ring, ring_bytes, fz_it, abort_flag,
      [&](int, int i, const uint8_t* src) {
        float a = 0.f;
#pragma unroll
        for (int k = 0; k < KC; ++k) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + k * 2048);
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            a = fmaf(xv[k * kFuseCols + 2 * j], __uint_as_float(u[j] << 16), a);
            a = fmaf(xv[k * kFuseCols + 2 * j + 1], __uint_as_float(u[j] & 0xffff0000u), a);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) fs.red[q][i] = a;
      },
      [&](int r0, int n) {
        epi_sync();  // the batch's partial dots are in
        if (tid < n) {
          const float u = ((fs.red[0][tid] + fs.red[1][tid]) + fs.red[2][tid]) + fs.red[3][tid];
          fs.h[r0 + tid][0] = __bfloat162float(__float2bfloat16_rn(fs.h[r0 + tid][0] * u));
        }
      });
  if (!ok) return;
  fuse_rows_bulk<1, KC>(p, ui, fs, R, tid, ring, ring_bytes, fz_it, abort_flag);
}

// A kPathFused unit after its epilogue, every epilogue warp: compaction, the
// down projection of the active rows (with the gate score also their up
// projection), and a barrier that frees the scratch. uni / hv: this warp's
// union word and its lane's h values (token t in hv[t]; SiLU(g) for a
// gate-only unit); a warp whose wait failed passes uni = 0. last: the CTA
// has no further unit (the ring may be used for bulk copies of the rows).
__device__ __forceinline__ void fuse_unit(const GateUpTcParams& p, const UnitInfo& ui,
                                          FuseScratch& fs, uint32_t uni,
                                          const float (&hv)[kFuseTokens], int q, int lane,
                                          bool last, uint8_t* ring, uint32_t ring_bytes,
                                          volatile int* abort_flag) {
  const int m = ui.gr.m;
  const int R = fuse_compact(fs, uni, hv, m, q, lane);
  const int tid = 32 * q + lane;
  uint32_t fz_it = 0;  // one fused unit per CTA: the half barriers start here
  const int d = p.dm.d;
  const bool bulk = last && ring_bytes >= 4u * static_cast<uint32_t>(d) &&
                    (d == 4096 || d == 2048 || d == 1024);
  if (ui.gate_only) {
    // the host fuses gate-score units only as a CTA's last work, for one-token
    // groups and these widths; anything else is an internal error
    if (!(bulk && m == 1)) {
      report_error(p.ws.status, kErrDeviceInvalid);
    } else if (R > 0) {
      if (d == 4096) fuse_updown_bulk<4>(p, ui, fs, R, tid, ring, ring_bytes, fz_it, abort_flag);
      else if (d == 2048) fuse_updown_bulk<2>(p, ui, fs, R, tid, ring, ring_bytes, fz_it, abort_flag);
      else fuse_updown_bulk<1>(p, ui, fs, R, tid, ring, ring_bytes, fz_it, abort_flag);
    }
    if (tid == 0) {  // W_up rows this unit read
      atomicAdd(p.ws.counters + kCntUpRows, static_cast<unsigned long long>(R));
      atomicAdd(p.ws.counters + kCntFusedUpRows, static_cast<unsigned long long>(R));
    }
  } else if (R > 0) {
    if (bulk && m <= 2 && d == 4096) {
      if (m == 1) fuse_rows_bulk<1, 4>(p, ui, fs, R, tid, ring, ring_bytes, fz_it, abort_flag);
      else fuse_rows_bulk<2, 4>(p, ui, fs, R, tid, ring, ring_bytes, fz_it, abort_flag);
    } else if (bulk && m <= 2 && d == 2048) {
      fuse_rows_bulk<2, 2>(p, ui, fs, R, tid, ring, ring_bytes, fz_it, abort_flag);
    } else if (bulk && m <= 2 && d == 1024) {
      fuse_rows_bulk<2, 1>(p, ui, fs, R, tid, ring, ring_bytes, fz_it, abort_flag);
    } else if (m == 1 && d % 4096 == 0) {
      fuse_cols<1, 4>(p, ui, fs, R, tid);
    } else if (m <= 2 && d % 2048 == 0) {
      fuse_cols<2, 2>(p, ui, fs, R, tid);
    } else if (m == 1) {
      fuse_cols<1, 1>(p, ui, fs, R, tid);
    } else if (m == 2) {
      fuse_cols<2, 1>(p, ui, fs, R, tid);
    } else {
      fuse_cols<4, 1>(p, ui, fs, R, tid);
    }
  }
  if (tid == 0) {  // W_down rows this unit read
    atomicAdd(p.ws.counters + kCntDownRows, static_cast<unsigned long long>(R));
    atomicAdd(p.ws.counters + kCntFusedRows, static_cast<unsigned long long>(R));
  }
  epi_sync();
}

// One-token routing in every CTA (dm.route1), all threads, before the warp
// roles start: the token's logits against every router row (a warp per
// expert, lanes over d, eight 16-byte loads of each in flight; scratch: the
// first stage of the weight ring, unused until the roles start), its top-k
// (topk_warp, as the routers pick), and the selected experts in expert order
// as the groups, one token each. The first CTA also writes what the router
// would have written for the getters and the combine (top-k ids and weights,
// slots, groups, paths, counters, meta), zeroes the output accumulator row,
// and then publishes meta[kMetaRoute1]; the other CTAs wait for it before
// their first atomic add (their epilogue, many microseconds later).
__device__ void route1_prologue(const GateUpTcParams& p, float* lg, Route1Groups& r1, int warp,
                                int lane) {
  const int E = p.dm.E, d = p.dm.d, k = p.dm.k;
  for (int e = warp; e < E; e += kThreads / 32) {
    const __nv_bfloat16* wr = p.wr + static_cast<size_t>(e) * d;
    float a = 0.f;
    for (int c0 = lane * 8; c0 < d; c0 += 32 * 8 * 8) {
      uint4 wv[8], xv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + u * 32 * 8;
        wv[u] = c < d ? __ldg(reinterpret_cast<const uint4*>(wr + c)) : make_uint4(0u, 0u, 0u, 0u);
        xv[u] = c < d ? __ldg(reinterpret_cast<const uint4*>(p.x + c)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t wa[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
        const uint32_t xa[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          a = fmaf(__uint_as_float(xa[j] << 16), __uint_as_float(wa[j] << 16), a);
          a = fmaf(__uint_as_float(xa[j] & 0xffff0000u), __uint_as_float(wa[j] & 0xffff0000u), a);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) lg[e] = a + (p.rbias ? p.rbias[e] : 0.f);
  }
  __syncthreads();
  if (warp == 0) {
    const TopkResult r = topk_warp(lg, E, k, lane);
    const float w = p.dm.renorm ? r.my_p / r.psum : r.my_p;
    int rank = 0;  // position of this lane's expert in expert order (ids are distinct)
    for (int j = 0; j < k; ++j) {
      const int ej = __shfl_sync(0xffffffffu, r.my_e, j);
      if (lane < k && ej < r.my_e) ++rank;
    }
    if (lane < k) {
      r1.exp[rank] = r.my_e;
      r1.w[rank] = w;
    }
    if (lane == 0) r1.k = k;
    if (blockIdx.x == 0 && lane < k) {
      const int slot = rank * kSlotAlign;
      p.ws.topk_idx[lane] = r.my_e;
      p.ws.topk_w[lane] = w;
      p.ws.slot_of[lane] = slot;
      p.ws.slot_w[slot] = w;
      p.ws.perm[slot] = 0;
      for (int q = 1; q < kSlotAlign; ++q) p.ws.perm[slot + q] = -1;
      Group gr;
      gr.expert = r.my_e;
      gr.slot0 = slot;
      gr.m = 1;
      gr.xrow0 = slot;
      p.ws.groups[rank] = gr;
      p.ws.group_path[rank] = kPathFused;
      p.ws.union_cnt[rank] = 0;
    }
  }
  if (blockIdx.x == 0) {
    const int tid = threadIdx.x;
    if (tid < kCntWords) {
      unsigned long long v = 0ull;
      if (tid == kCntGemv) v = static_cast<unsigned long long>(k);  // fused row-stream groups
      if (tid == kCntRoutedH) v = static_cast<unsigned long long>(k) * p.dm.F;
      p.ws.counters[tid] = v;
    }
    if (tid == 0) {
      p.ws.meta[kMetaGroups] = k;
      p.ws.meta[kMetaRoutedGroups] = k;
      p.ws.meta[kMetaSlotsUsed] = k * kSlotAlign;
      p.ws.meta[kMetaExpertsTouched] = k;
      p.ws.meta[kMetaGemvCount] = 0;
      p.ws.meta[kMetaTcCount] = 0;
      p.ws.meta[kMetaDone] = 0;
      p.ws.meta[kMetaTcQueue] = 0;
    }
    float4* y4 = reinterpret_cast<float4*>(p.ws.y);  // the output accumulator row
    for (int i = tid; i < d / 4; i += kThreads) y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    __threadfence();
    __syncthreads();
    if (tid == 0)
      asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p.ws.meta + kMetaRoute1), "r"(1)
                   : "memory");
  }
  __syncthreads();
}

// Two CTAs per SM for groups of <= 32 tokens: at most 168 registers a thread.
__global__ void __launch_bounds__(kThreads, 2)
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
  FuseScratch* fscr = reinterpret_cast<FuseScratch*>(
      (reinterpret_cast<uintptr_t>(tmem_slot) + 16 + 15) & ~static_cast<uintptr_t>(15));

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
    if (p.dm.fuse_down) {
      mbar_init(&fscr->bar[0], 1);
      mbar_init(&fscr->bar[1], 1);
    }
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

  const Route1Groups* r1 = nullptr;
  if (p.dm.route1) {
    route1_prologue(p, reinterpret_cast<float*>(smem), fscr->r1, warp, lane);
    r1 = &fscr->r1;
  }
  const int n_rg = r1 ? r1->k : __ldcg(p.ws.meta + kMetaRoutedGroups);
  const int n_g = r1 ? r1->k : __ldcg(p.ws.meta + kMetaGroups);
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
      }
      if (p.dm.S > 0 || r1) tma_prefetch_desc(&p.tm_x);
    }
    uint32_t it = 0;
    bool ok = true;
    Segs sg = segs_begin(n_units, KB, split);
    int u, kb0, kb1;
    while (ok && segs_next(sg, u, kb0, kb1)) {
      const UnitInfo ui = decode_unit(p, u, n_rg, tiles_r, tiles_s, r1);
      const int N = (ui.gr.m + 15) & ~15;
      const int nb = N / kBRowBox;
      const CUtensorMap* mg = ui.shared ? &p.tm_wgs : &p.tm_wg;
      const CUtensorMap* mu = ui.shared ? &p.tm_wus : &p.tm_wu;
      const CUtensorMap* mx = ui.shared || r1 ? &p.tm_x : &p.tm_xperm;
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
      const UnitInfo ui = decode_unit(p, u, n_rg, tiles_r, tiles_s, r1);
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
    // routing in this kernel: the first CTA's records (and zeroed counters)
    // are in place before this warp's first atomic add
    if (r1 && blockIdx.x != 0) {
      if (lane == 0 && !wait_flag(p.ws.meta + kMetaRoute1, abort_flag, p.ws.status)) ok = false;
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    Segs sg = segs_begin(n_units, KB, split);
    int u, kb0, kb1;
    for (; segs_next(sg, u, kb0, kb1); ++uidx) {
      // every epilogue warp walks every segment (named barriers below), doing
      // nothing once a wait has failed
      const UnitInfo ui = decode_unit(p, u, n_rg, tiles_r, tiles_s, r1);
      const int g = group_of_unit(u, n_rg, tiles_r, tiles_s);
      const int m = ui.gr.m;
      const int N = (m + 15) & ~15;
      const uint32_t b = uidx % p.nbuf;
      const uint32_t tph = (uidx / p.nbuf) & 1u;
      if (ok && !warp_wait(tfull + b, tph, abort_flag, p.ws.status)) ok = false;
      const bool whole = kb0 == 0 && kb1 == KB;
      const bool last_part = !whole && kb1 == KB;
      uint32_t uni = 0;       // this warp's union word (fused down projection)
      float hv[kFuseTokens];  // this lane's masked h of the first tokens
#pragma unroll
      for (int i = 0; i < kFuseTokens; ++i) hv[i] = 0.f;
      if (ok) {
        tc_fence_after();
        const float tau = ui.shared ? p.tau_shared : p.tau;
        const int row_i = 32 * q + lane;
        const int j = ui.nt * kNeuronTile + row_i;  // neuron of this thread
        const int word = (ui.nt * kNeuronTile + 32 * q) >> 5;
        __nv_bfloat16* row = ht + static_cast<size_t>(j) * ld + ui.gr.slot0;
        const uint32_t tg = tmem_base + lane_off + b * buf_cols;
        const uint32_t tu = tg + n_max;
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
            float hc[16];
            epi_chunk(p, ui, word, c0, m, tau, gv, uv, row, uni, nact, lane, hc);
            if (c0 == 0)
#pragma unroll
              for (int i = 0; i < kFuseTokens; ++i) hv[i] = hc[i];
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
      // the TMEM buffer is back with the MMA warp: the next unit's tiles
      // stream while this one's active W_down rows are read
      if (whole && ui.fused) {
        Segs rest = sg;  // no segment and no parked unit after this one: the ring is idle
        int u2, a2, b2;
        const bool last = park_u < 0 && !segs_next(rest, u2, a2, b2);
        fuse_unit(p, ui, *fscr, ok ? uni : 0u, hv, q, lane, last, smem, stages * stage_bytes,
                  abort_flag);
      }
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
        const UnitInfo ui = decode_unit(p, park_u, n_rg, tiles_r, tiles_s, r1);
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
        float hv[kFuseTokens];
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
          float hc[16];
          epi_chunk(p, ui, word, c0, m, tau, gv, uv, row, uni, nact, lane, hc);
          if (c0 == 0)
#pragma unroll
            for (int i = 0; i < kFuseTokens; ++i) hv[i] = hc[i];
        }
        epi_finish(p, ui, g, word, uni, nact, lane);
        if (q == 0 && lane == 0)
          atomicAdd(p.ws.counters + kCntGateUpRows, (ui.gate_only ? 1ull : 2ull) * kNeuronTile);
        if (ui.fused)
          fuse_unit(p, ui, *fscr, uni, hv, q, lane, true, smem, stages * stage_bytes, abort_flag);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
  // direct combine with no row-stream launch after this one: the last CTA
  // writes out from the accumulator rows
  if (p.dm.fuse_finish) direct_finish(p.dm, p.ws, p.out, p.out_bf16);
}

}  // namespace

size_t gate_up_tc_smem_bytes(int n_max, int stages, int b_blocks, bool fuse) {
  const size_t stage_bytes = 2 * kABytes + static_cast<size_t>(b_blocks) * n_max * 128;
  return 1024 + stages * stage_bytes + (2 * stages + 5) * sizeof(uint64_t) + 16 +
         (fuse ? 16 + sizeof(FuseScratch) : 0);
}

cudaError_t launch_gate_up_tc(const GateUpTcParams& p, int grid, size_t smem, cudaStream_t st) {
  // the launch's own size: the kernel has a little static shared memory too,
  // and the opt-in limit covers both
  const cudaError_t e = smem_limit(gate_up_tc_kernel, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(gate_up_tc_kernel, grid, kThreads, smem, st, p);
}

}  // namespace moe
