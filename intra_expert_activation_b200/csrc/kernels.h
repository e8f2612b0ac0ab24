// Internal interface between the C-ABI host code and the kernels: layer
// dimensions, workspace pointers, kernel parameter blocks, launch wrappers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace moe {

// Every kernel is launched with programmatic stream serialization: its
// launch is set up while the previous kernel on the stream drains (its CTAs
// are scheduled as the predecessor's CTAs exit), and they call
// grid_dep_wait() (griddepcontrol.wait) before touching global memory, so
// part of the launch latency overlaps the predecessor's tail. MOE_PDL=0 in
// the environment turns it off.
bool pdl_enabled();

template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device. The attribute is per device, so it is set once per
// (kernel, device) and remembered under a lock: contexts on several devices
// of one process, or on several threads, each get it.
cudaError_t smem_limit_at_least(const void* kernel, int bytes);
template <typename... KArgs>
cudaError_t smem_limit(void (*kernel)(KArgs...), int bytes) {
  return smem_limit_at_least(reinterpret_cast<const void*>(kernel), bytes);
}

constexpr uint32_t kSpinLimit = 4u << 20;  // ~1 s of polling with backoff
constexpr int kErrDeviceInvalid = 1;       // == MOE_ERR_INVALID: an internal consistency check failed
constexpr int kErrDeviceTimeout = 5;       // == MOE_ERR_DEVICE_TIMEOUT

constexpr int kGroupMax = 128;      // tokens per expert token group (gate/up tile N)
// Decode batches of 33-64 tokens whose experts average at most 16 tokens
// (Mixtral-shaped T = 64: 128 pairs over 8 experts) cap their groups at this
// many tokens, so that gate/up runs 32-column tiles at two CTAs per SM; an
// expert with more tokens becomes two groups (its weights are read twice).
constexpr int kGroupMaxDecode = 32;
constexpr int kGatherMaxTokens = 64;  // groups on the gathered TC path hold <= 64 tokens
constexpr int kSlotAlign = 8;       // expert slot ranges start at multiples of 8 slots
constexpr int kNeuronTile = 128;    // gate/up neurons per MMA tile (M)
constexpr int kDownSlice = 128;     // d_model columns per down TC tile (M)
constexpr int kKBlock = 64;         // K elements per pipeline stage (128 B of bf16)
constexpr int kRouteTokens = 16;    // tokens per router CTA
constexpr int kListMax = 2048;      // expert token groups per forward at most
constexpr int kGemvTokens = 8;      // tokens per GEMV pass (the row-stream mma's N)
// AUTO with the |h| score: groups of gemv_max < m <= kGemvCandMax tokens
// (one GEMV pass) choose their down path after gate/up from the size of
// their active-row union: the row stream if passes x union rows <=
// kCandNum / kCandDen x d_ff, else all rows on the tensor cores. The ratio is
// the measured bandwidth of the row stream over that of the all-rows
// tensor-core path on the Mixtral-shaped layer (about 5.0 and 6.3 TB/s per
// launch, CUDA-event timed).
constexpr int kGemvCandMax = 8;
constexpr int kCandNum = 4, kCandDen = 5;
// AUTO and DENSE: when at least kTcJoinNum / kTcJoinDen of a batch's groups
// take the tensor-core path by their size alone (more than gemv_cand
// tokens) and all of the batch's groups fit the tensor-core grid in one wave,
// the batch's smaller groups join them there (all rows) instead of starting
// the row-stream kernel for a few groups. Measured on the Mixtral-shaped
// layer at T = 32 (groups of 4, 5, 8, 8, 9, 9, 10, 11 tokens): 466 us per
// layer with all eight on the tensor cores against 485 us with the two
// smallest on the row stream (the row-stream launch and its start-up cost
// more than the extra rows, which take otherwise idle CTAs). With more
// groups than the grid holds (128 small experts, T = 256) the joiners' rows
// cost their full time: 272 vs 268 us, so that case keeps the row stream.
constexpr int kTcJoinNum = 1, kTcJoinDen = 2;

// A candidate group (kPathCand) takes the row stream when its passes over
// the union rows cost less than all F_e rows on the tensor cores; both down
// kernels evaluate it on the union count the gate/up epilogue left.
__host__ __device__ inline bool cand_takes_gemv(int union_rows, int passes, int F_e) {
  return static_cast<long long>(union_rows) * passes * kCandDen <=
         static_cast<long long>(F_e) * kCandNum;
}

// meta[] words written by the router's scan
enum Meta { kMetaGroups = 0, kMetaRoutedGroups = 1, kMetaDone = 2, kMetaSlotsUsed = 3,
            kMetaExpertsTouched = 4, kMetaGemvCount = 5, kMetaTcCount = 6,
            kMetaDownDone = 7,  // row-stream CTAs finished (direct combine ticket)
            kMetaTcQueue = 8,   // next tensor-core down unit to hand out
            kMetaRoute1 = 9,    // one-token routing in the gate/up kernel: layout published
            kMetaWords = 16 };

// counters[] (u64), reset by the router's scan every forward
enum Counter { kCntRoutedActive = 0, kCntSharedActive = 1, kCntDownRows = 2, kCntGemv = 3,
               kCntTcGather = 4, kCntTc = 5, kCntRoutedH = 6, kCntSharedH = 7,
               kCntUpRows = 8, kCntGateUpRows = 9, kCntGemvRows = 10, kCntFusedRows = 11,
               kCntFusedUpRows = 12, kCntWords = 13 };

// kPathCand: GEMV or all-rows TC, chosen after gate/up (cand_takes_gemv).
// kPathFused: a row-stream group whose down projection the gate/up kernel
// does itself, per 128-neuron tile, right after the tile's epilogue
// (Dims::fuse_down); it is on neither down kernel's list.
enum GroupPath { kPathNone = 0, kPathGemv = 1, kPathTcGather = 2, kPathTcAll = 3, kPathCand = 4,
                 kPathFused = 5 };

// Groups of at most kFuseTokens tokens on the row stream are fused into the
// gate/up kernel when Dims::fuse_down is set.
constexpr int kFuseTokens = 4;

// Requested path (mirrors moe_path in the public header).
enum Mode { kModeAuto = 0, kModeDense = 1, kModeGemv = 2, kModeTc = 3, kModeTcAll = 4 };

// One expert token group: up to kGroupMax consecutive slots of one expert.
struct Group {
  int32_t expert;  // 0..E-1 routed; E + s for shared expert s
  int32_t slot0;   // first slot: column of H^T and row of Y
  int32_t m;       // tokens in the group
  int32_t xrow0;   // first row of the activations: X_perm row (routed) or token (shared)
};

struct Dims {
  int d, F, Fs, E, S, k, T, renorm;
  int F_max;          // max(F, Fs)
  int fw;             // 32-bit words per neuron bitmap row: F_max / 32 (rounded up)
  int slots_routed;   // routed slot capacity (multiple of kSlotAlign)
  int slots_total;    // routed + shared slots = leading dimension of H^T
  int T_pad;          // tokens rounded up to kSlotAlign (per shared expert)
  int groups_max;
  int mode;           // Mode
  int gemv_max;       // AUTO: GEMV for groups with m <= gemv_max
  int gemv_cand;      // AUTO: groups with gemv_max < m <= gemv_cand are candidates
  float gather_density;
  int no_tc;          // 1: no tensor-core down path (fp32 layers): every group on GEMV
  int n_sms;          // streaming multiprocessors of the device
  int sk_ctas;        // capacity of the gate/up split-unit flags (CTAs), 0: no split units
  int score_gate;     // 1: active iff |SiLU(g)| > tau
  int sparse_up;      // 1 (gate score, tau > 0): GEMV groups compute the up projection only
                      // for their active rows (gate-only GEMM, then the fused up + down
                      // row stream); 0: the up projection is dense
  int tc_grid;        // CTAs of this forward's tensor-core down launch
  int tc_part_units;  // capacity of the tensor-core down part buffers (units), 0: none
  // 1: every group of this forward is on the row stream (and T <= kDirectMax):
  // the row stream adds w x its sums straight into the output accumulator
  // rows Y[0..T) (zeroed by the router) and its last CTA writes out; no
  // combine launch
  int direct_combine;
  // 1: row-stream groups of <= kFuseTokens tokens (one token with the gate
  // score's sparse up projection) take kPathFused: the gate/up kernel
  // multiplies each tile's active W_down rows (with the gate score first the
  // W_up rows) by its h values and adds the sums into Y (bf16 layers)
  int fuse_down;
  // 1 (with direct_combine): no row-stream launch follows the gate/up kernel,
  // so its last CTA (a ticket) writes out from the accumulator rows
  int fuse_finish;
  // 1: a one-token batch with no shared experts whose whole layer runs in the
  // gate/up kernel: every CTA routes the token itself (logits, top-k; the
  // selected experts in expert order are the groups, one token each), the
  // first CTA also writes the routing records, and no router launches
  int route1;
  // tokens per group at most in this forward: kGroupMax, or kGroupMaxDecode
  // (group_cap); the router's groups and every launch's tile width follow it
  int gcap;
};

// The group cap of a forward (Dims::gcap) from the layer's capacity record
// (E, S, no_tc) and the batch.
__host__ __device__ inline int group_cap(const Dims& cap, int T, int k) {
  if (!cap.no_tc && cap.S == 0 && T > kGroupMaxDecode && T <= 2 * kGroupMaxDecode &&
      2 * T * k <= kGroupMaxDecode * cap.E)
    return kGroupMaxDecode;
  return kGroupMax;
}

constexpr int kDirectMax = 16;  // tokens up to which the row stream combines directly

// K parts per tensor-core down unit (group, 128-column slice). A unit reads
// all of its group's rows for its columns, and an SM streams at most about
// 35-40 GB/s, so HBM is only saturated when every SM has work: with few
// groups most SMs idled (one 117 MB group of the Mixtral-shaped layer = 32
// units took 108 us). When the units fill less than 3/4 of the grid, each
// unit's rows are cut into ks parts, enough for about two units per CTA,
// ks = ceil(2 grid / units) (at most kTcMaxParts, at least one K-block per
// part, and within dm.tc_part_units part units); the CTAs take units from a
// queue (an atomic ticket), so the units of the SMs that stream slower are
// taken over by the others. Parts write fp32 partial sums to the workspace
// and the last part of a unit to finish (a ticket) adds them in part order
// into Y, so results do not depend on timing. Only groups of <=
// kTcPartTokens tokens are cut (decode batches). The router (to clear the
// tickets) and the kernel evaluate it on the same inputs.
constexpr int kTcMaxParts = 24;
constexpr int kTcPartTokens = 64;
__host__ __device__ inline int tc_ksplit(const Dims& dm, int n_tc) {
  if (n_tc <= 0 || dm.tc_grid <= 0 || dm.tc_part_units <= 0) return 1;
  const int tmax = dm.T < dm.gcap ? dm.T : dm.gcap;
  if ((tmax + 15) / 16 * 16 > kTcPartTokens) return 1;
  const long long grid = dm.tc_grid;
  const long long base = static_cast<long long>(n_tc) * (dm.d / kDownSlice);
  // forced gathered rows: the units' lengths follow their groups' unions,
  // so they are always cut (the queue then evens out the CTAs)
  if (dm.mode != kModeTc && 4 * base >= 3 * grid) return 1;
  const int f_min = dm.S > 0 && dm.Fs < dm.F ? dm.Fs : dm.F;
  long long ks = (2 * grid + base - 1) / base;
  if (ks > kTcMaxParts) ks = kTcMaxParts;
  if (ks > f_min / kKBlock) ks = f_min / kKBlock;
  if (ks > dm.tc_part_units / base) ks = dm.tc_part_units / base;
  return ks < 1 ? 1 : static_cast<int>(ks);
}

struct Workspace {
  int* status;                  // [1] device error word
  int* meta;                    // [kMetaWords]
  unsigned long long* counters; // [kCntWords]
  int* topk_idx;                // [Tmax*kmax]
  float* topk_w;                // [Tmax*kmax]
  int* slot_of;                 // [Tmax*kmax]
  int* rank_cta;                // [Tmax*kmax] rank of a pair among its CTA's pairs of that expert
  int* hist;                    // [E][router CTAs] per-CTA expert counts, then CTA base offsets
  int* expert_off;              // [E+1] first slot of each expert (multiple of kSlotAlign)
  int* expert_cnt;              // [E] routed pairs per expert
  int* perm;                    // [slots_routed] token of each routed slot, -1 for padding
  Group* groups;                // [groups_max]
  int* group_path;              // [groups_max]
  uint32_t* union_bits;         // [groups_max][fw]
  int* union_cnt;               // [groups_max] rows in each group's union (cleared by the router,
                                //   accumulated by the gate/up epilogue)
  int* gemv_list;               // [groups_max] groups on the GEMV path (count in meta)
  int* tc_list;                 // [groups_max] groups on a tensor-core path (count in meta)
  int* y_zero;                  // [E+1] 1: expert's Y rows (last: shared experts') start at zero
  float* slot_w;                // [slots_routed] combine weight of each routed slot
  int* sk_flags;                // [sk_ctas] gate/up: CTA c published its split-unit partial
  float* sk_part;               // [2 * sk_ctas][2][128][n_max] gate/up split-unit partial sums
  int* tc_ticket;               // [tc_part_units] parts of a TC down unit done (cleared by the router)
  float* tc_part;               // [tc_part_units][kTcPartTokens][128] TC down part sums

  uint32_t* act_bits;           // [slots_total][fw] or null (debug off)
  void* xperm;                  // [slots_routed][d] activations gathered by slot
  void* ht;                     // [F_max][slots_total] masked h, transposed
  float* y;                     // [slots_total][d] per-slot expert outputs
};

// ------------------------------------------------------------ gate + up (tcgen05)
struct GateUpTcParams {
  CUtensorMap tm_wg, tm_wu;    // [E*F][d], box {64, 128}
  CUtensorMap tm_wgs, tm_wus;  // [S*Fs][d], box {64, 128}
  CUtensorMap tm_xperm;        // [slots_routed][d], box {64, 16}
  CUtensorMap tm_x;            // [T][d], box {64, 16}
  Dims dm;
  Workspace ws;
  float tau, tau_shared;
  int dense;                   // 1: no threshold
  int n_max;                   // largest MMA N of this launch (multiple of 16, <= 256)
  int stages;
  int nbuf;                    // TMEM accumulator buffers (1 or 2)
  uint32_t tmem_cols;          // allocated TMEM columns
  int split;                   // 1: the leftover units after whole rounds are cut along K
  int b_blocks;                // activation regions per stage: 2 with the gate score, else 1
  const __nv_bfloat16* wd;     // [E*F][d] W_down (fused down projection, kPathFused groups)
  const __nv_bfloat16* wds;    // [S*Fs][d] shared experts' W_down
  const __nv_bfloat16* wu;     // [E*F][d] W_up (gate score: fused up + down of one-token groups)
  const __nv_bfloat16* wus;    // [S*Fs][d] shared experts' W_up
  const __nv_bfloat16* x;      // [T][d] the layer input (shared experts' tokens)
  const __nv_bfloat16* wr;     // [E][d] W_router (dm.route1)
  const float* rbias;          // [E] router bias or null (dm.route1)
  void* out;                   // [T][d] layer output (dm.fuse_finish)
  int out_bf16;                // out's type: 1 bf16, 0 fp32
};

// ------------------------------------------------------------ down (tcgen05)
struct DownTcParams {
  CUtensorMap tm_wd_blk;   // [E*F][d], box {64,64}
  CUtensorMap tm_wds_blk;  // [S*Fs][d]
  CUtensorMap tm_ht_blk;   // [F_max][slots_total], box {64,64}
  const void* wd;          // the same three arrays for the gathered rows' 16-byte copies
  const void* wds;
  const void* ht;
  Dims dm;
  Workspace ws;
  int n_max;        // largest MMA N of this launch
  int stages;
  uint32_t tmem_cols;
  int b_bytes;      // B bytes per stage
};

cudaError_t launch_route(const Dims& dm, const Workspace& ws, const void* x, const void* Wr,
                         const float* bias, bool bf16, cudaStream_t st);
// True when one CTA does routing and the permute copies (launch_permute is then skipped).
bool route_is_small(const Dims& dm);
cudaError_t launch_permute(const Dims& dm, const Workspace& ws, const void* x, bool bf16,
                           cudaStream_t st);
cudaError_t launch_gate_up_tc(const GateUpTcParams& p, int grid, size_t smem, cudaStream_t st);
// Dynamic shared memory of a gate/up launch; `fuse`: room for the fused
// down projection's row list and h values.
size_t gate_up_tc_smem_bytes(int n_max, int stages, int b_blocks, bool fuse);
cudaError_t launch_updown_gemv(const Dims& dm, const Workspace& ws, const void* Wu,
                               const void* Wus, const void* Wd, const void* Wds, const void* x,
                               bool bf16, int n_sms, cudaStream_t st);
cudaError_t launch_gate_up_simt(const Dims& dm, const Workspace& ws, const float* x,
                                const float* Wg, const float* Wu, const float* Wgs,
                                const float* Wus, float tau, float tau_shared, int dense,
                                cudaStream_t st);
cudaError_t launch_union_scan(const Dims& dm, const Workspace& ws, cudaStream_t st);
cudaError_t launch_down_gemv(const Dims& dm, const Workspace& ws, const void* Wd,
                             const void* Wds, bool bf16, int n_sms, void* out, bool out_bf16,
                             cudaStream_t st);
cudaError_t launch_down_tc(const DownTcParams& p, int grid, size_t smem, cudaStream_t st);
size_t down_tc_smem_bytes(int b_bytes, int stages, int fw);
cudaError_t launch_combine(const Dims& dm, const Workspace& ws, void* out, bool bf16,
                           cudaStream_t st);
#if defined(MOE_CHECK) && MOE_CHECK
// Checked build: a one-CTA kernel whose bounded wait (0: mbarrier, 1: global
// flag) never completes and gives up after `limit` probes.
cudaError_t launch_wait_timeout(int* status, uint32_t limit, int which, cudaStream_t st);
#endif
cudaError_t launch_debug_gather(const Dims& dm, const Workspace& ws, int32_t* topk_idx,
                                float* topk_w, uint32_t* bits, uint32_t* bits_shared,
                                cudaStream_t st);

}  // namespace moe
