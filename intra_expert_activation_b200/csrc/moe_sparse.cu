// C-ABI of the intra-expert sparse MoE layer: argument checking, the device
// workspace, the TMA descriptor cache and the launch sequence of one forward
//   route -> permute -> gate_up -> union_scan -> down (GEMV and/or TC) -> combine
// all on the caller's stream, with no allocation and no host synchronisation.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "kernels.h"
#include "moe_sparse.h"
#if defined(MOE_CHECK) && MOE_CHECK
#include "moe_sparse_check.h"
#endif

using moe::Dims;
using moe::Workspace;

namespace moe {
void set_last_error(const std::string& msg);
cudaError_t smem_limit_at_least(const void* kernel, int bytes) {
  struct Set {
    const void* kernel;
    int device, bytes;
  };
  static std::mutex mu;
  static std::vector<Set> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (Set& s : done)
    if (s.kernel == kernel && s.device == dev) {
      if (s.bytes >= bytes) return cudaSuccess;
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e == cudaSuccess) s.bytes = bytes;
      return e;
    }
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back({kernel, dev, bytes});
  return e;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("MOE_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

// Gate/up split units (MOE_GATE_UP_SPLIT=0 turns them off; a scheduling
// choice, the results are the same up to fp32 summation order).
bool split_enabled() {
  static const bool on = [] {
    const char* v = getenv("MOE_GATE_UP_SPLIT");
    return !(v && v[0] == '0');
  }();
  return on;
}

// One-token routing inside the gate/up kernel (MOE_FUSE_ROUTE=0 turns it off
// and launches the router, for comparisons).
bool fuse_route_enabled() {
  static const bool on = [] {
    const char* v = getenv("MOE_FUSE_ROUTE");
    return !(v && v[0] == '0');
  }();
  return on;
}

// Down projection of the smallest row-stream groups inside the gate/up kernel
// (MOE_FUSE_DOWN=0 turns it off and sends them to the row-stream kernel, for
// comparisons).
bool fuse_enabled() {
  static const bool on = [] {
    const char* v = getenv("MOE_FUSE_DOWN");
    return !(v && v[0] == '0');
  }();
  return on;
}
}  // namespace moe

namespace {

constexpr int kStages = 8;
const char* kStageNames[kStages] = {"route",       "permute",   "gate_up", "union_scan",
                                    "updown_gemv", "down_gemv", "down_tc", "combine"};
// NVTX ranges (no-ops unless a profiler is attached): one per forward, one
// per stage, so that a profiler can select the layer's launches by name
const char* kNvtxNames[kStages] = {"moe.route",       "moe.permute",   "moe.gate_up",
                                   "moe.union_scan",  "moe.updown_gemv", "moe.down_gemv",
                                   "moe.down_tc",     "moe.combine"};
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
// The stage range that is open: mark(i) closes the previous stage's range
// and opens stage i's; whatever is still open closes with the forward.
struct NvtxStages {
  bool open = false;
  void next(int i) {
    if (open) nvtxRangePop();
    open = i < kStages;
    if (open) nvtxRangePushA(kNvtxNames[i]);
  }
  ~NvtxStages() {
    if (open) nvtxRangePop();
  }
};

thread_local std::string g_init_error;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool get_encoder(std::string& err) {
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                                   cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
    err = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

// 2-D bf16 tensor map, 128-byte swizzle, out-of-range elements read as zero.
bool encode2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_in, uint32_t box_out, std::string& err) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_in, box_out};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d) for a [%llu][%llu] map", (int)r,
             (unsigned long long)outer, (unsigned long long)inner);
    err = buf;
    return false;
  }
  return true;
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
int roundup(int v, int a) { return (v + a - 1) / a * a; }
uint32_t pow2_at_least(uint32_t v) {
  uint32_t p = 32;
  while (p < v) p <<= 1;
  return p;
}
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Layout {
  Dims cap;
  size_t off[32];
  size_t total;
  long long sk_cols = 0;  // gate/up split partials: capacity in CTAs x MMA N (columns)
};

enum Buf { bStatus, bMeta, bCounters, bTopkIdx, bTopkW, bSlotOf, bRankCta, bHist, bExpOff,
           bExpCnt, bPerm, bGroups, bGroupPath,
           bUnionBits, bUnionCnt, bGemvList, bTcList, bYZero, bSlotW, bSkFlags, bSkPart,
           bTcTicket, bTcPart, bActBits, bXperm, bHt, bY, bCount };

moe_status check_desc(const moe_sparse_desc* d, std::string& err) {
  if (!d) { err = "desc is NULL"; return MOE_ERR_INVALID; }
  const bool bf16 = d->dtype == MOE_BF16;
  if (d->dtype != MOE_BF16 && d->dtype != MOE_F32) { err = "dtype must be MOE_F32 or MOE_BF16"; return MOE_ERR_INVALID; }
  if (d->d_model <= 0 || d->d_ff <= 0 || d->n_experts <= 0 || d->top_k_max <= 0 || d->max_tokens <= 0) {
    err = "d_model, d_ff, n_experts, top_k_max and max_tokens must be positive";
    return MOE_ERR_INVALID;
  }
  if (d->n_experts > 256) { err = "n_experts > 256"; return MOE_ERR_UNSUPPORTED; }
  if (d->top_k_max > d->n_experts || d->top_k_max > 16) { err = "top_k_max must be <= min(n_experts, 16)"; return MOE_ERR_INVALID; }
  if (d->max_tokens > 65536) { err = "max_tokens > 65536"; return MOE_ERR_UNSUPPORTED; }
  if (d->n_shared < 0 || d->n_shared > 8) { err = "n_shared must be in 0..8"; return MOE_ERR_INVALID; }
  const int dmod = bf16 ? 256 : 128, fmod = bf16 ? 128 : 32;
  if (d->d_model % dmod) { err = bf16 ? "d_model must be a multiple of 256 for bf16" : "d_model must be a multiple of 128 for fp32"; return MOE_ERR_UNSUPPORTED; }
  if (d->d_ff % fmod) { err = bf16 ? "d_ff must be a multiple of 128 for bf16" : "d_ff must be a multiple of 32 for fp32"; return MOE_ERR_UNSUPPORTED; }
  if (d->d_model > 32768 || d->d_ff > 65536) { err = "d_model > 32768 or d_ff > 65536"; return MOE_ERR_UNSUPPORTED; }
  if (d->n_shared > 0) {
    if (d->d_ff_shared <= 0 || d->d_ff_shared % fmod || d->d_ff_shared > 65536) {
      err = "d_ff_shared must be positive, <= 65536 and divisible like d_ff";
      return MOE_ERR_UNSUPPORTED;
    }
  }
  if (d->path < MOE_PATH_AUTO || d->path > MOE_PATH_SPARSE_TC_ALLROWS) { err = "unknown path"; return MOE_ERR_INVALID; }
  if (d->score != MOE_SCORE_H && d->score != MOE_SCORE_GATE) { err = "unknown score"; return MOE_ERR_INVALID; }
  if (d->out_f32 != 0 && d->out_f32 != 1) { err = "out_f32 must be 0 or 1"; return MOE_ERR_INVALID; }
  if (!bf16 && (d->path == MOE_PATH_SPARSE_TC || d->path == MOE_PATH_SPARSE_TC_ALLROWS)) {
    err = "tensor-core down paths need bf16";
    return MOE_ERR_UNSUPPORTED;
  }
  if (d->gemv_max_tokens < 0 || d->gemv_max_tokens > 256) { err = "gemv_max_tokens must be in 0..256"; return MOE_ERR_INVALID; }
  if (!(d->gather_max_density >= 0.f && d->gather_max_density <= 1.f)) { err = "gather_max_density must be in [0, 1]"; return MOE_ERR_INVALID; }
  if ((long long)d->max_tokens * d->top_k_max > (1ll << 22)) { err = "max_tokens * top_k_max > 2^22"; return MOE_ERR_UNSUPPORTED; }
  {
    const long long P = (long long)d->max_tokens * d->top_k_max;
    const long long groups = P / 128 + std::min<long long>(d->n_experts, P) +
                             (long long)d->n_shared * ((d->max_tokens + 127) / 128) + 1;
    if (groups > 2048) { err = "too many expert token groups (max_tokens * top_k_max too large)"; return MOE_ERR_UNSUPPORTED; }
  }
  return MOE_OK;
}

Layout make_layout(const moe_sparse_desc* d) {
  Layout L;
  Dims& c = L.cap;
  memset(&c, 0, sizeof c);
  const bool bf16 = d->dtype == MOE_BF16;
  c.d = d->d_model;
  c.F = d->d_ff;
  c.S = d->n_shared;
  c.Fs = c.S > 0 ? d->d_ff_shared : c.F;
  c.E = d->n_experts;
  c.k = d->top_k_max;
  c.T = d->max_tokens;
  c.renorm = d->renormalize ? 1 : 0;
  c.F_max = std::max(c.F, c.S > 0 ? c.Fs : 0);
  c.fw = (c.F_max + 31) / 32;
  const int P = c.T * c.k;
  c.slots_routed = roundup(P + (moe::kSlotAlign - 1) * std::min(c.E, P), moe::kSlotAlign);
  c.T_pad = roundup(c.T, moe::kSlotAlign);
  c.slots_total = c.slots_routed + c.S * c.T_pad;
  // groups at most: whole groups of the forward's cap plus one partial group
  // per touched expert (the cap is kGroupMaxDecode only for T <= 64)
  {
    auto bound = [&](int T_, int cap_) {
      const int P_ = T_ * c.k;
      return P_ / cap_ + std::min(c.E, P_) + c.S * ((T_ + cap_ - 1) / cap_) + 1;
    };
    c.groups_max = std::max(bound(c.T, moe::kGroupMax),
                            bound(std::min(c.T, 2 * moe::kGroupMaxDecode), moe::kGroupMaxDecode));
  }
  c.gcap = moe::kGroupMax;
  c.mode = d->path;
  c.gemv_max = d->gemv_max_tokens > 0 ? d->gemv_max_tokens : 4;
  // automatic threshold: groups of 5..kGemvCandMax tokens choose after gate/up
  c.gemv_cand = d->gemv_max_tokens == 0 && bf16 && d->path == MOE_PATH_AUTO &&
                        d->score != MOE_SCORE_GATE
                    ? moe::kGemvCandMax
                    : c.gemv_max;
  c.gather_density = d->gather_max_density;
  c.no_tc = bf16 ? 0 : 1;
  c.score_gate = d->score == MOE_SCORE_GATE ? 1 : 0;

  const size_t es = bf16 ? 2 : 4;
  size_t sz[bCount];
  sz[bStatus] = 64;
  sz[bMeta] = sizeof(int) * moe::kMetaWords;
  sz[bCounters] = sizeof(unsigned long long) * moe::kCntWords;
  sz[bTopkIdx] = sizeof(int) * P;
  sz[bTopkW] = sizeof(float) * P;
  sz[bSlotOf] = sizeof(int) * P;
  sz[bRankCta] = sizeof(int) * P;
  sz[bHist] = sizeof(int) * (size_t)((c.T + 1) / 2) * c.E;  // at most ceil(T/2) router CTAs
  sz[bExpOff] = sizeof(int) * (c.E + 1);
  sz[bExpCnt] = sizeof(int) * c.E;
  sz[bPerm] = sizeof(int) * c.slots_routed;
  sz[bGroups] = sizeof(moe::Group) * c.groups_max;
  sz[bGroupPath] = sizeof(int) * c.groups_max;
  sz[bUnionBits] = sizeof(uint32_t) * c.groups_max * c.fw;
  sz[bUnionCnt] = sizeof(int) * c.groups_max;
  sz[bGemvList] = sizeof(int) * c.groups_max;
  sz[bTcList] = sizeof(int) * c.groups_max;
  sz[bYZero] = sizeof(int) * (c.E + 1);
  sz[bSlotW] = sizeof(float) * c.slots_routed;
  // gate/up split units (bf16): one flag per CTA and two partial slots per CTA
  // of MMA N columns each: 2 x 160 CTAs (2 per SM) for groups of <= 32 tokens,
  // 160 CTAs for larger ones (cut only up to 64 tokens)
  {
    const int nm = std::min(roundup(std::min(c.T, moe::kGroupMax), 16), 64);
    c.sk_ctas = bf16 ? 320 : 0;
    L.sk_cols = bf16 ? std::max(320LL * std::min(nm, 32), 160LL * nm) : 0;
    sz[bSkFlags] = sizeof(int) * (size_t)c.sk_ctas;
    sz[bSkPart] = sizeof(float) * (size_t)2 * L.sk_cols * 2 * moe::kNeuronTile;
  }
  // tensor-core down units cut along K (bf16, groups of <= 64 tokens): a
  // ticket per unit and a partial-sum block per part unit
  c.tc_part_units = bf16 ? 1024 : 0;
  sz[bTcTicket] = sizeof(int) * (size_t)c.tc_part_units;
  sz[bTcPart] = sizeof(float) * (size_t)c.tc_part_units * moe::kTcPartTokens * moe::kDownSlice;
  sz[bActBits] = d->debug ? sizeof(uint32_t) * (size_t)c.slots_total * c.fw : 0;
  sz[bXperm] = es * (size_t)c.slots_routed * c.d;
  sz[bHt] = es * (size_t)c.F_max * c.slots_total;
  sz[bY] = sizeof(float) * (size_t)c.slots_total * c.d;
  size_t o = 0;
  for (int i = 0; i < bCount; ++i) {
    L.off[i] = o;
    o += align256(sz[i]);
  }
  L.total = o;
  return L;
}

struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

}  // namespace

void moe::set_last_error(const std::string& msg) { g_init_error = msg; }

struct moe_sparse_ctx {
  moe_sparse_desc desc;
  Layout lay;
  bool bf16 = false;
  int n_sms = 0;
  void* mem = nullptr;
  Workspace ws;
  // shared experts
  const void* Wgs = nullptr;
  const void* Wus = nullptr;
  const void* Wds = nullptr;
  float tau_shared = 0.f;
  bool shared_set = false;
  // tensor-map cache (bf16 layers)
  const void* c_wg = nullptr;
  const void* c_wu = nullptr;
  const void* c_wd = nullptr;
  const void* c_x = nullptr;
  int c_xT = -1;
  bool maps_shared_ok = false;
  CUtensorMap tm_wg, tm_wu, tm_wgs, tm_wus, tm_xperm, tm_x;
  CUtensorMap tm_wd_blk, tm_wds_blk, tm_ht_blk;
  // last forward
  Dims last;
  bool has_last = false;
  // timing: a ring of event sets, one per timed forward
  int ring = 0;
  std::vector<cudaEvent_t> ev;             // ring * (kStages + 1)
  std::vector<uint8_t> ran;                // ring * kStages
  int64_t n_timed = 0;                     // timed forwards since the last collection
  int64_t next_set = 0;
  int last_set = -1;
  int64_t launches = 0;
  std::string err;
};

namespace {

moe_status fail(moe_sparse_ctx* c, moe_status s, const std::string& msg) {
  if (c) c->err = msg; else g_init_error = msg;
  return s;
}

moe_status cuda_fail(moe_sparse_ctx* c, cudaError_t e, const char* what) {
  std::string m = std::string(what) + ": " + cudaGetErrorString(e);
  return fail(c, MOE_ERR_CUDA, m);
}

bool build_weight_maps(moe_sparse_ctx* c, const void* Wg, const void* Wu, const void* Wd) {
  const Dims& k = c->lay.cap;
  const uint64_t rb = (uint64_t)k.d * 2;
  if (c->c_wg != Wg) {
    if (!encode2d(&c->tm_wg, Wg, k.d, (uint64_t)k.E * k.F, rb, 64, 128, c->err)) return false;
    c->c_wg = Wg;
  }
  if (c->c_wu != Wu) {
    if (!encode2d(&c->tm_wu, Wu, k.d, (uint64_t)k.E * k.F, rb, 64, 128, c->err)) return false;
    c->c_wu = Wu;
  }
  if (c->c_wd != Wd) {
    if (!encode2d(&c->tm_wd_blk, Wd, k.d, (uint64_t)k.E * k.F, rb, 64, 64, c->err)) return false;
    c->c_wd = Wd;
  }
  return true;
}

}  // namespace

extern "C" {

moe_status moe_sparse_validate_desc(const moe_sparse_desc* desc) {
  return check_desc(desc, g_init_error);
}

moe_status moe_sparse_workspace_bytes(const moe_sparse_desc* desc, size_t* bytes) {
  moe_status s = check_desc(desc, g_init_error);
  if (s != MOE_OK) return s;
  if (!bytes) { g_init_error = "bytes is NULL"; return MOE_ERR_INVALID; }
  *bytes = make_layout(desc).total;
  return MOE_OK;
}

moe_status moe_sparse_init(const moe_sparse_desc* desc, moe_sparse_ctx** out) {
  if (!out) { g_init_error = "ctx output pointer is NULL"; return MOE_ERR_INVALID; }
  *out = nullptr;
  moe_status s = check_desc(desc, g_init_error);
  if (s != MOE_OK) return s;
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess || ndev == 0) { g_init_error = "no CUDA device"; return MOE_ERR_CUDA; }
  if (desc->device < 0 || desc->device >= ndev) { g_init_error = "device ordinal out of range"; return MOE_ERR_INVALID; }
  DeviceGuard dg(desc->device);
  if (!dg.ok) { g_init_error = "cudaSetDevice failed"; return MOE_ERR_CUDA; }
  int major = 0, minor = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, desc->device);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, desc->device);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, desc->device);
  if (major != 10 || minor != 0) {
    g_init_error = "this library is built for sm_100a (B200); device is sm_" +
                   std::to_string(major) + std::to_string(minor);
    return MOE_ERR_UNSUPPORTED;
  }
  std::string err;
  if (!get_encoder(err)) { g_init_error = err; return MOE_ERR_CUDA; }

  moe_sparse_ctx* c = new moe_sparse_ctx();
  c->desc = *desc;
  c->lay = make_layout(desc);
  c->bf16 = desc->dtype == MOE_BF16;
  c->n_sms = sms;
  c->lay.cap.n_sms = sms;
  e = cudaMalloc(&c->mem, c->lay.total);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_init_error = "cudaMalloc of a " + std::to_string(c->lay.total) + "-byte workspace failed";
    delete c;
    return MOE_ERR_NOMEM;
  }
  e = cudaMemset(c->mem, 0, c->lay.total);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaFree(c->mem);
    delete c;
    g_init_error = std::string("workspace clear failed: ") + cudaGetErrorString(e);
    return MOE_ERR_CUDA;
  }
  uint8_t* b = static_cast<uint8_t*>(c->mem);
  const size_t* o = c->lay.off;
  Workspace& w = c->ws;
  w.status = reinterpret_cast<int*>(b + o[bStatus]);
  w.meta = reinterpret_cast<int*>(b + o[bMeta]);
  w.counters = reinterpret_cast<unsigned long long*>(b + o[bCounters]);
  w.topk_idx = reinterpret_cast<int*>(b + o[bTopkIdx]);
  w.topk_w = reinterpret_cast<float*>(b + o[bTopkW]);
  w.slot_of = reinterpret_cast<int*>(b + o[bSlotOf]);
  w.rank_cta = reinterpret_cast<int*>(b + o[bRankCta]);
  w.hist = reinterpret_cast<int*>(b + o[bHist]);
  w.expert_off = reinterpret_cast<int*>(b + o[bExpOff]);
  w.expert_cnt = reinterpret_cast<int*>(b + o[bExpCnt]);
  w.perm = reinterpret_cast<int*>(b + o[bPerm]);
  w.groups = reinterpret_cast<moe::Group*>(b + o[bGroups]);
  w.group_path = reinterpret_cast<int*>(b + o[bGroupPath]);
  w.union_bits = reinterpret_cast<uint32_t*>(b + o[bUnionBits]);
  w.union_cnt = reinterpret_cast<int*>(b + o[bUnionCnt]);
  w.gemv_list = reinterpret_cast<int*>(b + o[bGemvList]);
  w.tc_list = reinterpret_cast<int*>(b + o[bTcList]);
  w.y_zero = reinterpret_cast<int*>(b + o[bYZero]);
  w.slot_w = reinterpret_cast<float*>(b + o[bSlotW]);
  w.sk_flags = reinterpret_cast<int*>(b + o[bSkFlags]);
  w.sk_part = reinterpret_cast<float*>(b + o[bSkPart]);
  w.tc_ticket = reinterpret_cast<int*>(b + o[bTcTicket]);
  w.tc_part = reinterpret_cast<float*>(b + o[bTcPart]);
  w.act_bits = desc->debug ? reinterpret_cast<uint32_t*>(b + o[bActBits]) : nullptr;
  w.xperm = b + o[bXperm];
  w.ht = b + o[bHt];
  w.y = reinterpret_cast<float*>(b + o[bY]);

  if (c->bf16) {
    const Dims& k = c->lay.cap;
    bool ok = encode2d(&c->tm_xperm, w.xperm, k.d, k.slots_routed, (uint64_t)k.d * 2, 64, 16, err) &&
              encode2d(&c->tm_ht_blk, w.ht, k.slots_total, k.F_max, (uint64_t)k.slots_total * 2, 64, 64, err);
    if (!ok) {
      cudaFree(c->mem);
      delete c;
      g_init_error = err;
      return MOE_ERR_CUDA;
    }
    // unused maps still need a valid encoding (kernel parameters are copied whole)
    c->tm_wgs = c->tm_xperm;
    c->tm_wus = c->tm_xperm;
    c->tm_x = c->tm_xperm;
    c->tm_wds_blk = c->tm_ht_blk;
  }
  *out = c;
  return MOE_OK;
}

moe_status moe_sparse_set_shared(moe_sparse_ctx* c, const void* Wg_s, const void* Wu_s,
                                 const void* Wd_s, float tau_shared) {
  if (!c) return MOE_ERR_INVALID;
  if (c->desc.n_shared == 0) return fail(c, MOE_ERR_INVALID, "context has no shared experts");
  if (!Wg_s || !Wu_s || !Wd_s) return fail(c, MOE_ERR_INVALID, "shared weight pointer is NULL");
  if (!aligned16(Wg_s) || !aligned16(Wu_s) || !aligned16(Wd_s))
    return fail(c, MOE_ERR_INVALID, "shared weights must be 16-byte aligned");
  if (std::isnan(tau_shared)) return fail(c, MOE_ERR_INVALID, "tau_shared is NaN");
  if (c->bf16) {
    const Dims& k = c->lay.cap;
    const uint64_t rb = (uint64_t)k.d * 2, rows = (uint64_t)k.S * k.Fs;
    if (!encode2d(&c->tm_wgs, Wg_s, k.d, rows, rb, 64, 128, c->err) ||
        !encode2d(&c->tm_wus, Wu_s, k.d, rows, rb, 64, 128, c->err) ||
        !encode2d(&c->tm_wds_blk, Wd_s, k.d, rows, rb, 64, 64, c->err))
      return MOE_ERR_CUDA;
  }
  c->Wgs = Wg_s;
  c->Wus = Wu_s;
  c->Wds = Wd_s;
  c->tau_shared = tau_shared;
  c->shared_set = true;
  return MOE_OK;
}

moe_status moe_sparse_forward(moe_sparse_ctx* c, const void* x, int32_t T, const void* W_router,
                              const float* router_bias, const void* W_gate, const void* W_up,
                              const void* W_down, float tau, int32_t top_k, void* out,
                              void* stream) {
  if (!c) return MOE_ERR_INVALID;
  const Dims& cap = c->lay.cap;
  if (T < 0 || T > cap.T) return fail(c, MOE_ERR_INVALID, "T out of range [0, max_tokens]");
  if (top_k < 1 || top_k > cap.k) return fail(c, MOE_ERR_INVALID, "top_k out of range [1, top_k_max]");
  if (T == 0) return MOE_OK;
  if (!x || !W_router || !W_gate || !W_up || !W_down || !out)
    return fail(c, MOE_ERR_INVALID, "NULL tensor pointer");
  if (!aligned16(x) || !aligned16(W_router) || !aligned16(W_gate) || !aligned16(W_up) ||
      !aligned16(W_down) || !aligned16(out))
    return fail(c, MOE_ERR_INVALID, "tensors must be 16-byte aligned");
  if (router_bias && (reinterpret_cast<uintptr_t>(router_bias) & 3u))
    return fail(c, MOE_ERR_INVALID, "router_bias must be 4-byte aligned");
  if (std::isnan(tau)) return fail(c, MOE_ERR_INVALID, "tau is NaN");
  if (cap.S > 0 && !c->shared_set)
    return fail(c, MOE_ERR_INVALID, "shared experts declared but moe_sparse_set_shared not called");

  DeviceGuard dg(c->desc.device);
  if (!dg.ok) return fail(c, MOE_ERR_CUDA, "cudaSetDevice failed");
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  Dims dm = cap;
  dm.T = T;
  dm.k = top_k;
  const int P = T * top_k;
  dm.gcap = moe::group_cap(cap, T, top_k);
  dm.groups_max = P / dm.gcap + std::min(cap.E, P) + cap.S * ((T + dm.gcap - 1) / dm.gcap) + 1;
  const bool dense = c->desc.path == MOE_PATH_DENSE;
  const int mode = c->desc.path;
  const int tmax = std::min(T, dm.gcap);  // no group holds more tokens
  // AUTO only: tensor-core groups whose union is at most this fraction of
  // d_ff read only the union rows (the forced paths fix the rows they read)
  if (mode != MOE_PATH_AUTO) dm.gather_density = 0.f;
  // AUTO batches whose groups all fit one row-stream pass: every
  // group streams its union rows, the 5-8-token candidates included. The
  // candidate rule prices the tensor cores at their many-group rate; a batch
  // this small has at most T x k / 5 such groups, and a tensor-core launch
  // with one to three groups streams at 0.55-0.69 of HBM, below the row
  // stream's ~0.77. No tensor-core launch then. The combine stays a kernel
  // of its own for these batches: the row stream's direct combine (adds into
  // the token rows, the last CTA writing out) measured no faster with groups
  // of 5-8 tokens (T = 8 on the Mixtral-shaped layer: 95.0 us for the row
  // stream and the output, against 86.4 + 7.4 us for the row stream and the
  // combine launch).
  // The gate score, whose groups of more than 4 tokens otherwise take the
  // tensor cores by size, follows the same rule.
  const bool rs_only = mode == MOE_PATH_AUTO && c->bf16 && c->desc.gemv_max_tokens == 0 &&
                       tmax > cap.gemv_max && tmax <= moe::kGemvCandMax;
  if (rs_only) dm.gemv_max = moe::kGemvCandMax;
  bool need_gemv = !(mode == MOE_PATH_SPARSE_TC || mode == MOE_PATH_SPARSE_TC_ALLROWS) || !c->bf16;
  const bool need_tc = c->bf16 && mode != MOE_PATH_SPARSE_GEMV &&
                       !((mode == MOE_PATH_AUTO || mode == MOE_PATH_DENSE) && tmax <= dm.gemv_max);
  const int n_max = roundup(tmax, 16);
  // gate score: the GEMV groups' up projection is sparse (only the active
  // rows) when the threshold can leave rows out; at tau <= 0 every neuron
  // whose SiLU(g) is non-zero is active, so the dense up projection (gate and
  // up in one GEMM) reads the same rows faster
  dm.sparse_up = dm.score_gate && tau > 0.f ? 1 : 0;
  // gate/up units (group x 128-neuron tile) at most, and the launch's CTAs
  const int gu_units_max =
      (P / dm.gcap + std::min(cap.E, P)) * (cap.F / moe::kNeuronTile) +
      cap.S * ((T + dm.gcap - 1) / dm.gcap) * (cap.Fs / moe::kNeuronTile);
  const int gu_ctas_per_sm = n_max <= 32 ? 2 : 1;
  // (with fewer units than CTA slots, one unit per CTA: cutting the units
  // along K over the full grid to even out the SMs measured slower, 120 vs
  // 108 us per layer at T = 1 on the Mixtral-shaped layer)
  const int gu_grid = std::max(1, std::min(gu_units_max, gu_ctas_per_sm * c->n_sms));
  // row-stream groups of <= kFuseTokens tokens: down projection inside the
  // gate/up kernel (bf16, dense up projection, automatic or dense path), when
  // no CTA has more than one unit to finish, so that the down rows stream
  // after the CTA's weight tiles. With several units per CTA the down rows
  // would share HBM with the next units' tiles through 16-byte loads, which
  // stream slower than the row-stream kernel's bulk copies (measured at
  // T = 8 on the Mixtral-shaped layer: 384 vs 363 us per layer); with one
  // unit per CTA the fusion saves the row-stream launch and its start-up
  // (T = 1: 110 vs 120 us).
  // With the gate score (sparse up projection) the gate/up kernel also does
  // the up projection of the active rows of one-token groups, for rows of
  // 1, 2 or 4 KB (the layout of its bulk path).
  dm.fuse_down = c->bf16 && (mode == MOE_PATH_AUTO || mode == MOE_PATH_DENSE) &&
                 gu_units_max <= gu_grid &&
                 (!dm.sparse_up || cap.d == 1024 || cap.d == 2048 || cap.d == 4096) &&
                 moe::fuse_enabled() ? 1 : 0;
  if (dm.fuse_down) {
    // the row-stream kernel is only needed for groups the fusion leaves:
    // unfused row-stream groups and candidates
    const int fused_max = dm.sparse_up ? 1 : moe::kFuseTokens;
    const bool big_gemv = std::min(tmax, dm.gemv_max) > fused_max;
    const bool cand = dm.gemv_cand > dm.gemv_max && tmax > dm.gemv_max;
    need_gemv = big_gemv || cand;
  }
  // every group on a row stream (fused or not; with the gate score only when
  // all of them are fused, since its separate kernel has no direct combine)
  // and a small batch: the row stream combines directly into the output (no
  // combine launch); with no row-stream launch the gate/up kernel writes out
  const bool out_bf16 = c->bf16 && !c->desc.out_f32;
  dm.direct_combine = (need_gemv || dm.fuse_down) && !need_tc && !rs_only &&
                              (!dm.sparse_up || !need_gemv) && T <= moe::kDirectMax
                          ? 1
                          : 0;
  dm.fuse_finish = dm.direct_combine && !need_gemv ? 1 : 0;
  // one token, every group fused and combined directly, no shared experts, a
  // small router: the gate/up kernel routes the token itself in every CTA
  // (no router launch)
  dm.route1 = dm.fuse_finish && T == 1 && cap.S == 0 && top_k <= 16 &&
                      (size_t)cap.E * cap.d * 2 <= 64 * 1024 && moe::fuse_route_enabled()
                  ? 1
                  : 0;
  // the tensor-core down launch's grid is fixed here: the router's layout
  // and the kernel both derive the units' K parts from it
  const int tc_ctas_per_sm = n_max <= 64 ? 2 : 1;
  {
    const long long units_max =
        (long long)dm.groups_max * (cap.d / moe::kDownSlice) * moe::kTcMaxParts;
    dm.tc_grid = need_tc ? (int)std::max<long long>(
                               1, std::min<long long>(units_max, tc_ctas_per_sm * c->n_sms))
                         : 0;
  }

  if (c->bf16) {
    if (!build_weight_maps(c, W_gate, W_up, W_down)) return MOE_ERR_CUDA;
    if ((cap.S > 0 || dm.route1) && (c->c_x != x || c->c_xT != T)) {
      if (!encode2d(&c->tm_x, x, cap.d, (uint64_t)T, (uint64_t)cap.d * 2, 64, 16, c->err))
        return MOE_ERR_CUDA;
      c->c_x = x;
      c->c_xT = T;
    }
  }

  const bool timing = c->ring > 0;
  const int set = timing ? static_cast<int>(c->next_set % c->ring) : 0;
  cudaEvent_t* evs = timing ? &c->ev[static_cast<size_t>(set) * (kStages + 1)] : nullptr;
  uint8_t* ran = timing ? &c->ran[static_cast<size_t>(set) * kStages] : nullptr;
  bool stage_ran[kStages] = {};
  NvtxRange forward_range("moe.forward");
  NvtxStages stage_range;
  auto mark = [&](int i) {
    stage_range.next(i);
    if (timing) cudaEventRecord(evs[i], st);
  };
  cudaError_t e;
  mark(0);
  if (!dm.route1) {
    e = moe::launch_route(dm, c->ws, x, W_router, router_bias, c->bf16, st);
    if (e != cudaSuccess) return cuda_fail(c, e, "route launch");
    stage_ran[0] = true;
  }
  mark(1);
  if (!moe::route_is_small(dm)) {
    e = moe::launch_permute(dm, c->ws, x, c->bf16, st);
    if (e != cudaSuccess) return cuda_fail(c, e, "permute launch");
    stage_ran[1] = true;
  }
  mark(2);

  if (c->bf16) {
    moe::GateUpTcParams p;
    p.tm_wg = c->tm_wg;
    p.tm_wu = c->tm_wu;
    p.tm_wgs = c->tm_wgs;
    p.tm_wus = c->tm_wus;
    p.tm_xperm = c->tm_xperm;
    p.tm_x = c->tm_x;
    p.dm = dm;
    p.ws = c->ws;
    p.tau = tau;
    p.tau_shared = c->tau_shared;
    p.dense = dense ? 1 : 0;
    p.n_max = n_max;
    const uint32_t buf = 2u * n_max;
    p.nbuf = 2 * buf <= 512 ? 2 : 1;
    p.tmem_cols = pow2_at_least(p.nbuf * buf);
    const size_t budget = gu_ctas_per_sm == 2 ? 113 * 1024 : 225 * 1024;
    // gate score: gate-only units take two K-blocks per stage; the second
    // activation region costs a stage of the pipeline when groups are larger
    // than 16 tokens (measured at T = 32: 303 -> 358 us), so only below that
    p.b_blocks = dm.sparse_up && n_max <= 16 ? 2 : 1;
    const size_t stage_bytes = 32768 + (size_t)p.b_blocks * n_max * 128;
    const size_t fuse_bytes =
        moe::gate_up_tc_smem_bytes(n_max, 0, p.b_blocks, dm.fuse_down) -
        moe::gate_up_tc_smem_bytes(n_max, 0, p.b_blocks, false);
    p.stages = (int)std::min<size_t>(8, (budget - 2048 - fuse_bytes) / stage_bytes);
    const size_t smem = moe::gate_up_tc_smem_bytes(n_max, p.stages, p.b_blocks, dm.fuse_down);
    p.wd = static_cast<const __nv_bfloat16*>(W_down);
    p.wds = static_cast<const __nv_bfloat16*>(c->Wds);
    p.wu = static_cast<const __nv_bfloat16*>(W_up);
    p.wus = static_cast<const __nv_bfloat16*>(c->Wus);
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.wr = static_cast<const __nv_bfloat16*>(W_router);
    p.rbias = router_bias;
    p.out = out;
    p.out_bf16 = out_bf16 ? 1 : 0;
    const int grid = gu_grid;
    // leftover units are cut along K only for groups of <= 64 tokens: with
    // 128-token groups (prefill) the parts' accumulators cost more than the
    // uneven last round (measured: +24 us at T = 4096, d = 2048)
    p.split = moe::split_enabled() && n_max <= 64 && grid <= cap.sk_ctas &&
                      (long long)grid * n_max <= c->lay.sk_cols
                  ? 1
                  : 0;
    e = moe::launch_gate_up_tc(p, grid, smem, st);
  } else {
    e = moe::launch_gate_up_simt(dm, c->ws, static_cast<const float*>(x),
                                 static_cast<const float*>(W_gate), static_cast<const float*>(W_up),
                                 static_cast<const float*>(c->Wgs), static_cast<const float*>(c->Wus),
                                 tau, c->tau_shared, dense ? 1 : 0, st);
  }
  if (e != cudaSuccess) return cuda_fail(c, e, "gate_up launch");
  stage_ran[2] = true;
  mark(3);
  if (c->desc.path == MOE_PATH_SPARSE_TC) {  // only the gathered path needs row lists
    e = moe::launch_union_scan(dm, c->ws, st);
    if (e != cudaSuccess) return cuda_fail(c, e, "union_scan launch");
    stage_ran[3] = true;
  }
  mark(4);

  if (need_gemv && dm.sparse_up) {  // GEMV groups: fused sparse up + down over the active rows
    e = moe::launch_updown_gemv(dm, c->ws, W_up, c->Wus, W_down, c->Wds, x, c->bf16, c->n_sms,
                                st);
    if (e != cudaSuccess) return cuda_fail(c, e, "updown_gemv launch");
    stage_ran[4] = true;
  }
  mark(5);
  if (need_gemv && !dm.sparse_up) {
    e = moe::launch_down_gemv(dm, c->ws, W_down, c->Wds, c->bf16, c->n_sms, out, out_bf16, st);
    if (e != cudaSuccess) return cuda_fail(c, e, "down_gemv launch");
    stage_ran[5] = true;
  }
  mark(6);
  if (need_tc) {
    moe::DownTcParams p;
    p.tm_wd_blk = c->tm_wd_blk;
    p.tm_wds_blk = c->tm_wds_blk;
    p.wd = W_down;
    p.wds = c->Wds;
    p.ht = c->ws.ht;
    p.dm = dm;
    p.ws = c->ws;
    p.n_max = n_max;
    p.tm_ht_blk = c->tm_ht_blk;
    p.b_bytes = std::max(8192, (n_max + 63) / 64 * 8192);
    p.tmem_cols = pow2_at_least(2u * n_max);
    // small groups (decode): two CTAs per SM so that a unit's epilogue and
    // the next unit's loads overlap across CTAs; large groups: one CTA
    // (per SM 228 KB, of which each CTA's static shared memory and 1 KB the
    // system reserves)
    const size_t budget = tc_ctas_per_sm == 2 ? 113 * 1024 - 128 : 225 * 1024;
    p.stages = 8;
    while (p.stages > 2 && moe::down_tc_smem_bytes(p.b_bytes, p.stages, dm.fw) > budget) --p.stages;
    const size_t smem = moe::down_tc_smem_bytes(p.b_bytes, p.stages, dm.fw);
    e = moe::launch_down_tc(p, dm.tc_grid, smem, st);
    if (e != cudaSuccess) return cuda_fail(c, e, "down_tc launch");
    stage_ran[6] = true;
  }
  mark(7);
  if (!dm.direct_combine) {
    e = moe::launch_combine(dm, c->ws, out, out_bf16, st);
    if (e != cudaSuccess) return cuda_fail(c, e, "combine launch");
    stage_ran[7] = true;
  }
  mark(8);
  int nl = 0;
  for (int i = 0; i < kStages; ++i) nl += stage_ran[i];
  c->launches += nl;
  if (timing) {
    for (int i = 0; i < kStages; ++i) ran[i] = stage_ran[i];
    c->last_set = set;
    ++c->next_set;
    ++c->n_timed;
  }
  c->last = dm;
  c->has_last = true;
  return MOE_OK;
}

moe_status moe_sparse_get_debug(moe_sparse_ctx* c, int32_t* topk_idx, float* topk_w,
                                uint32_t* active_bits, uint32_t* active_bits_shared,
                                void* stream) {
  if (!c) return MOE_ERR_INVALID;
  if (!c->has_last) return fail(c, MOE_ERR_INVALID, "no forward has run");
  if ((active_bits || active_bits_shared) && !c->desc.debug)
    return fail(c, MOE_ERR_INVALID, "active bitmaps need desc.debug = 1");
  DeviceGuard dg(c->desc.device);
  cudaError_t e = moe::launch_debug_gather(c->last, c->ws, topk_idx, topk_w, active_bits,
                                           active_bits_shared, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(c, e, "debug gather launch");
  return MOE_OK;
}

moe_status moe_sparse_get_stats(moe_sparse_ctx* c, moe_stats* s, void* stream) {
  if (!c || !s) return MOE_ERR_INVALID;
  if (!c->has_last) return fail(c, MOE_ERR_INVALID, "no forward has run");
  DeviceGuard dg(c->desc.device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned long long cnt[moe::kCntWords];
  int meta[moe::kMetaWords];
  cudaError_t e = cudaMemcpyAsync(cnt, c->ws.counters, sizeof cnt, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(meta, c->ws.meta, sizeof meta, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(c, e, "stats copy");
  s->n_routed_h = (int64_t)cnt[moe::kCntRoutedH];
  s->n_routed_active = (int64_t)cnt[moe::kCntRoutedActive];
  s->n_shared_h = (int64_t)cnt[moe::kCntSharedH];
  s->n_shared_active = (int64_t)cnt[moe::kCntSharedActive];
  s->down_rows_read = (int64_t)cnt[moe::kCntDownRows];
  s->n_groups = meta[moe::kMetaGroups];
  s->n_groups_gemv = (int64_t)cnt[moe::kCntGemv];
  s->n_groups_tc_gather = (int64_t)cnt[moe::kCntTcGather];
  s->n_groups_tc_allrows = (int64_t)(cnt[moe::kCntTc] - cnt[moe::kCntTcGather]);
  s->n_experts_touched = meta[moe::kMetaExpertsTouched];
  s->up_rows_read = (int64_t)cnt[moe::kCntUpRows];
  s->gate_up_rows_read = (int64_t)cnt[moe::kCntGateUpRows];
  s->down_rows_gemv = (int64_t)cnt[moe::kCntGemvRows];
  s->down_rows_fused = (int64_t)cnt[moe::kCntFusedRows];
  s->up_rows_fused = (int64_t)cnt[moe::kCntFusedUpRows];
  return MOE_OK;
}

moe_status moe_sparse_get_status(moe_sparse_ctx* c, int32_t* device_err) {
  if (!c || !device_err) return MOE_ERR_INVALID;
  DeviceGuard dg(c->desc.device);
  cudaError_t e = cudaDeviceSynchronize();
  int v = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&v, c->ws.status, sizeof v, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(c->ws.status, 0, sizeof v);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(c, e, "status read");
  *device_err = v;
  return MOE_OK;
}

moe_status moe_sparse_set_timing(moe_sparse_ctx* c, int32_t ring) {
  if (!c || ring < 0 || ring > 4096) return MOE_ERR_INVALID;
  DeviceGuard dg(c->desc.device);
  for (cudaEvent_t e : c->ev)
    if (e) cudaEventDestroy(e);
  c->ev.assign(static_cast<size_t>(ring) * (kStages + 1), nullptr);
  c->ran.assign(static_cast<size_t>(ring) * kStages, 0);
  for (auto& e : c->ev) {
    cudaError_t r = cudaEventCreate(&e);
    if (r != cudaSuccess) {
      c->ring = 0;
      return cuda_fail(c, r, "event create");
    }
  }
  c->ring = ring;
  c->n_timed = 0;
  c->next_set = 0;
  c->last_set = -1;
  return MOE_OK;
}

static moe_status read_set(moe_sparse_ctx* c, int set, float* ms, int n) {
  cudaEvent_t* evs = &c->ev[static_cast<size_t>(set) * (kStages + 1)];
  const uint8_t* ran = &c->ran[static_cast<size_t>(set) * kStages];
  cudaError_t e = cudaEventSynchronize(evs[kStages]);
  if (e != cudaSuccess) return cuda_fail(c, e, "event sync");
  for (int i = 0; i < n && i < kStages; ++i) {
    float t = 0.f;
    if (ran[i]) {
      e = cudaEventElapsedTime(&t, evs[i], evs[i + 1]);
      if (e != cudaSuccess) return cuda_fail(c, e, "event elapsed");
    }
    ms[i] = t;
  }
  for (int i = kStages; i < n; ++i) ms[i] = 0.f;
  return MOE_OK;
}

moe_status moe_sparse_get_timing(moe_sparse_ctx* c, float* ms, int32_t n) {
  if (!c || !ms || n < 0) return MOE_ERR_INVALID;
  if (c->last_set < 0) return fail(c, MOE_ERR_INVALID, "no timed forward has run");
  DeviceGuard dg(c->desc.device);
  return read_set(c, c->last_set, ms, n);
}

moe_status moe_sparse_get_timing_all(moe_sparse_ctx* c, float* ms, int32_t n_stages,
                                     int32_t max_forwards, int32_t* n_forwards) {
  if (!c || !ms || !n_forwards || n_stages < 0 || max_forwards < 0) return MOE_ERR_INVALID;
  DeviceGuard dg(c->desc.device);
  int64_t avail = std::min<int64_t>(c->n_timed, c->ring);
  avail = std::min<int64_t>(avail, max_forwards);
  const int64_t first = c->next_set - avail;
  for (int64_t f = 0; f < avail; ++f) {
    const int set = static_cast<int>((first + f) % c->ring);
    moe_status s = read_set(c, set, ms + f * n_stages, n_stages);
    if (s != MOE_OK) return s;
  }
  *n_forwards = static_cast<int32_t>(avail);
  c->n_timed = 0;
  return MOE_OK;
}

moe_status moe_sparse_launch_count(const moe_sparse_ctx* c, int64_t* n) {
  if (!c || !n) return MOE_ERR_INVALID;
  *n = c->launches;
  return MOE_OK;
}

const char* moe_sparse_stage_name(int32_t i) {
  return (i >= 0 && i < kStages) ? kStageNames[i] : nullptr;
}

const char* moe_sparse_last_error(const moe_sparse_ctx* c) {
  return c ? c->err.c_str() : g_init_error.c_str();
}

#if defined(MOE_CHECK) && MOE_CHECK
moe_status moe_sparse_check_wait_timeout(moe_sparse_ctx* c, uint32_t limit, int32_t which,
                                         void* stream) {
  if (!c) return MOE_ERR_INVALID;
  if (which != 0 && which != 1) return fail(c, MOE_ERR_INVALID, "which must be 0 or 1");
  if (limit < 1 || limit > moe::kSpinLimit)
    return fail(c, MOE_ERR_INVALID, "limit must be in 1..kSpinLimit");
  DeviceGuard dg(c->desc.device);
  const cudaError_t e =
      moe::launch_wait_timeout(c->ws.status, limit, which, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(c, e, "wait_timeout launch");
  return MOE_OK;
}
#endif

moe_status moe_sparse_destroy(moe_sparse_ctx* c) {
  if (!c) return MOE_OK;
  {
    DeviceGuard dg(c->desc.device);
    for (cudaEvent_t e : c->ev)
      if (e) cudaEventDestroy(e);
    if (c->mem) cudaFree(c->mem);
  }
  delete c;
  return MOE_OK;
}

}  // extern "C"
