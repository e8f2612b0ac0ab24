// Router: logits, softmax over all experts, top-k (+ renormalisation), and a
// deterministic stable counting sort of the routed (token, expert) pairs into
// per-expert slot ranges and expert token groups. The pages keep the dense
// model's router as it is [gist.science EN "Uncovering Intra-expert
// Activation Sparsity for Efficient Mixture-of-Expert Model Execution",
// Technical Summary > Methodology > System Implementation in vLLM].
//
// route_kernel, one CTA per `tpc` tokens (2 at decode, up to kRouteTokens at
// prefill):
//   logits   the CTA's x rows are copied to shared memory; a warp takes 4
//            experts (and, with few experts, a slice of d) and keeps tpc x 4
//            fp32 sums in registers while its lanes stride d in 16-byte
//            vectors; butterfly reductions, a fixed summation order;
//   top-k    one warp per token: the k largest logits, equal logits to the
//            lower expert index; softmax weights, renormalised or not;
//   ranks    each pair's rank among the CTA's pairs of the same expert in
//            pair order (warp match + per-warp counts) and the CTA's
//            histogram hist[e][cta];
//   finish   the last CTA to finish (atomic ticket after a fence) turns the
//            histograms into per-CTA base offsets with one scan per expert
//            over the CTAs, pads each expert's slot range to kSlotAlign, and
//            lays out the token groups, their paths and the GEMV work.
// permute_kernel, one warp per pair: slot = expert_off[e] + base[cta][e] +
//   rank, so slots are ordered by (token, choice) within each expert; it
//   records perm / slot_of and copies the x row to X_perm[slot]; extra warps
//   mark the padding slots in perm (their X_perm rows are never used: every
//   kernel masks the columns of tokens past a group's count).
#include "common.cuh"
#include "topk.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxExperts = kTopkMaxExperts;
constexpr int kSmallTokens = 4;  // single-CTA routing (and permute) up to this batch

// 16-byte vectors of x / W_router rows, widened to fp32 (exactly).
template <typename TX>
struct XVec;
template <>
struct XVec<__nv_bfloat16> {
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
  __device__ static void load_shared(const __nv_bfloat16* p, float (&f)[8]) {
    unpack(*reinterpret_cast<const uint4*>(p), f);
  }
  __device__ static void load(const __nv_bfloat16* p, float (&f)[8]) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), f);
  }
};
template <>
struct XVec<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ static void load_shared(const float* p, float (&f)[4]) {
    unpack(*reinterpret_cast<const uint4*>(p), f);
  }
  __device__ static void load(const float* p, float (&f)[4]) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), f);
  }
};

// Path of a group from its token count and the requested mode (the
// batch-size switch of the pages, taken per expert token group).
__device__ __forceinline__ int group_path_of(const Dims& dm, int m) {
  if (dm.no_tc || dm.mode == kModeGemv) return kPathGemv;
  if (dm.mode == kModeTc) return kPathTcAll;  // gathered or not: decided by the union scan
  if (dm.mode == kModeTcAll) return kPathTcAll;
  if (m <= dm.gemv_max)  // auto and dense; the smallest groups inside the gate/up kernel
    return dm.fuse_down && m <= (dm.sparse_up ? 1 : kFuseTokens) ? kPathFused : kPathGemv;
  return m <= dm.gemv_cand ? kPathCand : kPathTcAll;
}

// Last CTA: histograms -> base offsets, expert slot ranges, token groups and
// the path of every group.
__device__ void build_layout(const Dims& dm, const Workspace& ws, const int* cnt, int* poff);

__device__ void route_finish(const Dims& dm, const Workspace& ws, int n_cta) {
  __shared__ int cnt[kMaxExperts];
  __shared__ int poff[kMaxExperts + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = dm.E;
  // per expert: exclusive scan of its CTA counts (contiguous, expert-major).
  // A warp takes kEb experts at a time and each lane 8 consecutive CTAs of a
  // 256-CTA chunk, so the loads of kEb experts' chunks are in flight together
  constexpr int kEb = 4;
  const int nw = blockDim.x / 32;
  for (int e0 = warp * kEb; e0 < E; e0 += nw * kEb) {
    int carry[kEb] = {};
    for (int c0 = 0; c0 < n_cta; c0 += 256) {
      int v[kEb][8];
#pragma unroll
      for (int j = 0; j < kEb; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c = c0 + lane * 8 + i;
          v[j][i] = (e0 + j < E && c < n_cta) ? __ldcg(ws.hist + (size_t)(e0 + j) * n_cta + c) : 0;
        }
#pragma unroll
      for (int j = 0; j < kEb; ++j) {
        int sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) sum += v[j][i];
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += u;
        }
        int run = carry[j] + incl - sum;
        if (e0 + j < E) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = c0 + lane * 8 + i;
            if (c < n_cta) ws.hist[(size_t)(e0 + j) * n_cta + c] = run;
            run += v[j][i];
          }
        }
        carry[j] += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    if (lane < kEb && e0 + lane < E) {
      int cv = carry[0];
#pragma unroll
      for (int j = 1; j < kEb; ++j)
        if (lane == j) cv = carry[j];
      cnt[e0 + lane] = cv;
    }
  }
  if (tid < kCntWords) ws.counters[tid] = 0ull;
  __syncthreads();
  build_layout(dm, ws, cnt, poff);
}

// Exclusive prefix sums over the CTA of N ints per thread, in thread order
// (v becomes the prefix, total the CTA-wide sums). sm: (32 + 1) * N ints.
// Every thread of the CTA calls it.
template <int N>
__device__ __forceinline__ void block_exclusive_scan(int (&v)[N], int (&total)[N], int* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int inc[N];
#pragma unroll
  for (int j = 0; j < N; ++j) inc[j] = v[j];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const int u = __shfl_up_sync(0xffffffffu, inc[j], o);
      if (lane >= o) inc[j] += u;
    }
  if (lane == 31)
#pragma unroll
    for (int j = 0; j < N; ++j) sm[warp * N + j] = inc[j];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const int w = lane < nw ? sm[lane * N + j] : 0;
      int wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += u;
      }
      if (lane < nw) sm[lane * N + j] = wi - w;
      if (lane == 31) sm[32 * N + j] = wi;
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < N; ++j) {
    v[j] = sm[warp * N + j] + inc[j] - v[j];
    total[j] = sm[32 * N + j];
  }
  __syncthreads();
}

// How one entry's tokens are cut into groups. An entry is a routed expert
// (q < E, its me = cnt[q] pairs) or a shared expert (q >= E, all T tokens):
__device__ __forceinline__ int on_gemv_list(int path) {
  return path == kPathGemv || path == kPathCand;
}
__device__ __forceinline__ int on_tc_list(int path) {
  return path == kPathTcAll || path == kPathTcGather || path == kPathCand;
}
// The group's Y rows receive atomic adds (row stream, fused or not), so they
// start at zero.
__device__ __forceinline__ int adds_into_y(int path) {
  return on_gemv_list(path) || path == kPathFused;
}

// ng groups of gsz tokens (a multiple of kSlotAlign; the last one has
// m_last), each at most dm.gcap (a multiple of kSlotAlign).
struct EntryCut {
  int me, ng, gsz, m_last, F_e, path_full, path_last;
};

// Whether a batch with n_groups groups, n_tc of them on the all-rows
// tensor-core path by their size alone, sends its row-stream groups there too:
// at least kTcJoinNum / kTcJoinDen of the groups are there already, and all
// groups' units (group x 128 output columns) fit the tensor-core launch's grid
// at once, so the joining groups take CTAs that would otherwise idle.
__device__ __forceinline__ bool tc_join(const Dims& dm, int n_tc, int n_groups) {
  return (dm.mode == kModeAuto || dm.mode == kModeDense) && !dm.no_tc && n_tc > 0 &&
         static_cast<long long>(n_tc) * kTcJoinDen >=
             static_cast<long long>(n_groups) * kTcJoinNum &&
         static_cast<long long>(n_groups) * (dm.d / kDownSlice) <= dm.tc_grid;
}
__device__ __forceinline__ int joined_path(int path, bool join) {
  return join && (path == kPathGemv || path == kPathCand || path == kPathFused) ? kPathTcAll
                                                                                : path;
}

__device__ __forceinline__ EntryCut entry_cut(const Dims& dm, const int* cnt, int q) {
  EntryCut c;
  c.me = q < dm.E ? cnt[q] : dm.T;
  c.F_e = q < dm.E ? dm.F : dm.Fs;
  if (c.me <= 0) {
    c.ng = c.gsz = c.m_last = 0;
    c.path_full = c.path_last = kPathGemv;
    return c;
  }
  const int n_g = (c.me + dm.gcap - 1) / dm.gcap;
  c.gsz = ((c.me + n_g - 1) / n_g + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
  c.ng = (c.me + c.gsz - 1) / c.gsz;
  c.m_last = c.me - (c.ng - 1) * c.gsz;
  c.path_full = group_path_of(dm, c.gsz);
  c.path_last = group_path_of(dm, c.m_last);
  return c;
}

// From the per-expert pair counts cnt[E] (shared memory): expert slot ranges
// poff[E+1] (shared), token groups, the path of every group, the GEMV and TC
// group lists, counters and meta; every group's union count is cleared for
// the gate/up epilogue to accumulate. Called by every thread of the CTA;
// counters must be zero. Each thread takes a run of consecutive entries
// (routed experts, then the shared experts); prefix sums over the CTA place
// their slots, groups and list entries, so group order is (expert, group) as
// in a serial walk over the experts.
__device__ void build_layout(const Dims& dm, const Workspace& ws, const int* cnt, int* poff) {
  constexpr int kPer = 2;  // entries per thread: E + S <= 264 <= 2 x 256 threads
  __shared__ int scan_sm[33 * 8];
  __shared__ int zero_shared;
  const int tid = threadIdx.x;
  const int E = dm.E, T = dm.T, k = dm.k, S = dm.S;
  const int n_ent = E + S;
  const int per = (n_ent + blockDim.x - 1) / blockDim.x;  // <= kPer
  const int q0 = min(tid * per, n_ent), q1 = min(q0 + per, n_ent);
  if (tid == 0) zero_shared = 0;

  // ---- pass 1: slots, groups, GEMV / TC list positions
  // kGemv / kTc: list lengths (a candidate group is in both lists); kCand:
  // candidates; kTcSharedDef: shared groups whose all-rows TC path is fixed now
  // kFused: groups whose down projection runs inside the gate/up kernel
  enum { kSlots, kGroups, kGemv, kTc, kCand, kRoutedGroups, kTcSharedDef, kTouched, kFused, kN };
  int v[kN] = {}, tot[kN];
  EntryCut cut[kPer];
  // ---- pass 0: groups, and those on the all-rows tensor-core path by size
  int g2[2] = {0, 0}, gt[2];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int q = q0 + i;
    if (q >= q1) continue;
    cut[i] = entry_cut(dm, cnt, q);
    const EntryCut& c = cut[i];
    if (c.ng == 0) continue;
    g2[0] += c.ng;
    g2[1] += (c.ng - 1) * (c.path_full == kPathTcAll) + (c.path_last == kPathTcAll);
  }
  block_exclusive_scan<2>(g2, gt, scan_sm);
  const bool join = tc_join(dm, gt[1], gt[0]);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int q = q0 + i;
    if (q >= q1) continue;
    cut[i].path_full = joined_path(cut[i].path_full, join);
    cut[i].path_last = joined_path(cut[i].path_last, join);
    const EntryCut c = cut[i];
    if (c.ng == 0) continue;
    const int n_gemv = (c.ng - 1) * on_gemv_list(c.path_full) + on_gemv_list(c.path_last);
    const int n_tc = (c.ng - 1) * on_tc_list(c.path_full) + on_tc_list(c.path_last);
    const int n_cand = (c.ng - 1) * (c.path_full == kPathCand) + (c.path_last == kPathCand);
    v[kFused] += (c.ng - 1) * (c.path_full == kPathFused) + (c.path_last == kPathFused);
    if (q < E) {
      v[kSlots] += (c.me + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
      v[kRoutedGroups] += c.ng;
      v[kTouched] += 1;
    } else {
      v[kTcSharedDef] += n_tc - n_cand;
    }
    v[kGroups] += c.ng;
    v[kGemv] += n_gemv;
    v[kTc] += n_tc;
    v[kCand] += n_cand;
  }
  block_exclusive_scan<kN>(v, tot, scan_sm);

  // ---- pass 2: write the groups and lists
  {
    int slot = v[kSlots], g = v[kGroups], gv = v[kGemv], tc = v[kTc];
    for (int i = 0; i < kPer; ++i) {
      const int q = q0 + i;
      if (q >= q1) continue;
      const EntryCut& c = cut[i];
      const bool routed = q < E;
      const int base = routed ? slot : dm.slots_routed + (q - E) * dm.T_pad;
      if (routed) poff[q] = slot;
      int any_gemv = 0;
      for (int j = 0; j < c.ng; ++j, ++g) {
        const int m = j == c.ng - 1 ? c.m_last : c.gsz;
        const int path = j == c.ng - 1 ? c.path_last : c.path_full;
        if (g < dm.groups_max) {
          Group gr;
          gr.expert = q;
          gr.slot0 = base + j * c.gsz;
          gr.m = m;
          gr.xrow0 = routed ? base + j * c.gsz : j * c.gsz;
          ws.groups[g] = gr;
          ws.group_path[g] = path;
          ws.union_cnt[g] = 0;
          any_gemv |= adds_into_y(path);
          if (on_gemv_list(path)) ws.gemv_list[gv++] = g;
          if (on_tc_list(path)) ws.tc_list[tc++] = g;
        }
      }
      if (routed) {
        ws.y_zero[q] = any_gemv;
        slot += (c.me + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
      } else if (any_gemv) {
        zero_shared = 1;  // benign race: every writer stores 1
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    poff[E] = tot[kSlots];
    ws.y_zero[E] = zero_shared;
    ws.meta[kMetaRoutedGroups] = tot[kRoutedGroups];
    ws.meta[kMetaGroups] = tot[kGroups];
    ws.meta[kMetaSlotsUsed] = tot[kSlots];
    ws.meta[kMetaExpertsTouched] = tot[kTouched];
    ws.meta[kMetaGemvCount] = tot[kGemv];
    ws.meta[kMetaTcCount] = tot[kTc];
    // candidates are counted by the down kernel that takes them
    ws.counters[kCntGemv] = tot[kGemv] - tot[kCand] + tot[kFused];
    ws.counters[kCntTc] = tot[kTc] - tot[kCand];
    if (dm.mode != kModeTc)  // the GEMV kernel adds its rows
      ws.counters[kCntDownRows] =
          (unsigned long long)(tot[kTc] - tot[kCand] - tot[kTcSharedDef]) * dm.F +
          (unsigned long long)tot[kTcSharedDef] * dm.Fs;
    ws.counters[kCntRoutedH] = (unsigned long long)T * k * (unsigned long long)dm.F;
    ws.counters[kCntSharedH] =
        (unsigned long long)S * (unsigned long long)T * (unsigned long long)dm.Fs;
    ws.meta[kMetaDone] = 0;      // ticket counter for the next forward
    ws.meta[kMetaDownDone] = 0;  // the row stream's direct-combine ticket
    ws.meta[kMetaTcQueue] = 0;   // the tensor-core down kernel's unit queue
  }
  __syncthreads();
  for (int x = tid; x <= E; x += blockDim.x) ws.expert_off[x] = poff[x];
  for (int x = tid; x < E; x += blockDim.x) ws.expert_cnt[x] = cnt[x];
  for (int x = tid; x < dm.sk_ctas; x += blockDim.x) ws.sk_flags[x] = 0;  // gate/up split units
  for (int x = tid; x < dm.tc_part_units; x += blockDim.x) ws.tc_ticket[x] = 0;  // TC down parts
}

// Dot product of one token row with one router row, lanes over d in chunks
// of 32 x VEC elements, loads issued in batches of kBatch chunks.
template <typename TX>
__device__ __forceinline__ float row_dot(const TX* a, const TX* b, int d, int lane) {
  constexpr int VEC = XVec<TX>::N;
  constexpr int kBatch = 8;
  float acc = 0.f;
  for (int c0 = lane * VEC; c0 < d; c0 += 32 * VEC * kBatch) {
    uint4 ra[kBatch], rb[kBatch];  // raw vectors: the loads of a batch are in flight together
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int c = c0 + i * 32 * VEC;
      if (c < d) {
        ra[i] = __ldg(reinterpret_cast<const uint4*>(a + c));
        rb[i] = __ldg(reinterpret_cast<const uint4*>(b + c));
      } else {
        ra[i] = rb[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      float av[VEC], bv[VEC];
      XVec<TX>::unpack(ra[i], av);
      XVec<TX>::unpack(rb[i], bv);
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc = fmaf(av[v], bv[v], acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// Top-k of one token's logits (one warp, topk_warp): the k largest, equal
// logits to the lower expert index; softmax over all experts; weights
// p / sum(p_sel) or p. Writes topk_idx / topk_w of token `tok`, the chosen
// experts to sel[0..k) and, if given, their weights to selw[0..k).
__device__ __forceinline__ void topk_token(const Dims& dm, const Workspace& ws, const float* lgt,
                                           int tok, int lane, int* sel, float* selw = nullptr) {
  const int k = dm.k;
  const TopkResult r = topk_warp(lgt, dm.E, k, lane);
  if (lane < k) {
    const float w = dm.renorm ? r.my_p / r.psum : r.my_p;
    ws.topk_idx[tok * k + lane] = r.my_e;
    ws.topk_w[tok * k + lane] = w;
    sel[lane] = r.my_e;
    if (selw) selw[lane] = w;
  }
}

// Logits of the CTA's tb <= TPC tokens, whose rows sit in shared memory in
// their stored type, against every expert. A warp item is (4 experts, one
// slice of d); its lanes stride the slice in 16-byte vectors and keep TPC x 4
// fp32 sums in registers, so one shared-memory vector of x feeds 4 experts
// and one W_router vector feeds all TPC tokens. With fewer than 4 x kWarps
// experts, d is split into up to kWarps / (E/4) slices so that every warp has
// work; the slices' sums are added in slice order (fixed summation order).
template <typename TX, int TPC>
__device__ __forceinline__ void staged_logits(const Dims& dm, const TX* xs, const TX* Wr,
                                              const float* bias, int tb,
                                              float (*lg)[kMaxExperts + 1], float* part) {
  constexpr int VEC = XVec<TX>::N;
  constexpr int EPW = 4;
  const int E = dm.E, d = dm.d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_eg = (E + EPW - 1) / EPW;
  const int ks = n_eg >= kWarps ? 1 : kWarps / n_eg;
  const int dsl = ((d / ks + VEC - 1) / VEC) * VEC;
  for (int item = warp; item < n_eg * ks; item += kWarps) {
    const int e0 = (item / ks) * EPW, s = item % ks;
    const int c0 = s * dsl, c1 = min(d, c0 + dsl);
    const TX* wrow[EPW];
#pragma unroll
    for (int j = 0; j < EPW; ++j) wrow[j] = Wr + (size_t)min(e0 + j, E - 1) * d;
    float acc[TPC][EPW];
#pragma unroll
    for (int t = 0; t < TPC; ++t)
#pragma unroll
      for (int j = 0; j < EPW; ++j) acc[t][j] = 0.f;
#pragma unroll(TPC <= 2 ? 4 : TPC <= 4 ? 2 : 1)
    for (int c = c0 + lane * VEC; c < c1; c += 32 * VEC) {
      float w[EPW][VEC];
#pragma unroll
      for (int j = 0; j < EPW; ++j) XVec<TX>::load(wrow[j] + c, w[j]);
#pragma unroll
      for (int t = 0; t < TPC; ++t) {
        if (t < tb) {
          float xv[VEC];
          XVec<TX>::load_shared(xs + (size_t)t * d + c, xv);
#pragma unroll
          for (int j = 0; j < EPW; ++j)
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[t][j] = fmaf(xv[v], w[j][v], acc[t][j]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TPC; ++t) {
#pragma unroll
      for (int j = 0; j < EPW; ++j) {
        float a = acc[t][j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        const int e = e0 + j;
        if (lane == 0 && t < tb && e < E) {
          if (ks == 1)
            lg[t][e] = a + (bias ? bias[e] : 0.f);
          else
            part[(s * TPC + t) * E + e] = a;
        }
      }
    }
  }
  if (ks > 1) {
    __syncthreads();
    for (int i = threadIdx.x; i < tb * E; i += kThreads) {
      const int t = i / E, e = i % E;
      float a = 0.f;
      for (int s = 0; s < ks; ++s) a += part[(s * TPC + t) * E + e];
      lg[t][e] = a + (bias ? bias[e] : 0.f);
    }
  }
}

template <typename TX, int TPC>
__global__ void __launch_bounds__(kThreads, 2) route_kernel(Dims dm, Workspace ws, const TX* x,
                                                            const TX* Wr, const float* bias,
                                                            int tpc, int stage_x) {
  __shared__ float lg[kRouteTokens][kMaxExperts + 1];
  __shared__ int sel[kRouteTokens * 16];
  __shared__ int wcnt[kWarps][kMaxExperts];
  __shared__ int is_last;

  grid_dep_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = dm.E, d = dm.d, T = dm.T, k = dm.k;
  const int tok0 = blockIdx.x * tpc;
  const int tb = min(tpc, T - tok0);

  if (stage_x) {
    // ---- logits with the CTA's x rows copied to shared memory as stored
    extern __shared__ __align__(16) uint8_t xs_raw[];
    TX* xs = reinterpret_cast<TX*>(xs_raw);  // [tb][d]
    const int nvec = tb * d * (int)sizeof(TX) / 16;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)tok0 * d);
    uint4* xs4 = reinterpret_cast<uint4*>(xs);
    constexpr int kV = 8;  // vectors per thread in flight together
    for (int base = 0; base < nvec; base += kThreads * kV) {
      uint4 r[kV];
#pragma unroll
      for (int i = 0; i < kV; ++i) {
        const int j = base + tid + kThreads * i;
        if (j < nvec) r[i] = __ldg(src + j);
      }
#pragma unroll
      for (int i = 0; i < kV; ++i) {
        const int j = base + tid + kThreads * i;
        if (j < nvec) xs4[j] = r[i];
      }
    }
    __syncthreads();
    // the split-d partial sums (slices x E <= 32, so at most 32 x TPC
    // floats) reuse wcnt, which is cleared only after the top-k
    static_assert(sizeof(wcnt) >= sizeof(float) * 32 * kRouteTokens, "partials");
    staged_logits<TX, TPC>(dm, xs, Wr, bias, tb, lg, reinterpret_cast<float*>(&wcnt[0][0]));
  } else {
    // ---- logits: warp tasks (token, expert), lanes over d
    for (int task = warp; task < tb * E; task += kWarps) {
      const int t = task / E, e = task % E;
      const float a = row_dot<TX>(x + (size_t)(tok0 + t) * d, Wr + (size_t)e * d, d, lane);
      if (lane == 0) lg[t][e] = a + (bias ? bias[e] : 0.f);
    }
  }
  __syncthreads();

  // ---- top-k and weights: one warp per token
  for (int t = warp; t < tb; t += kWarps)
    topk_token(dm, ws, lg[t], tok0 + t, lane, sel + t * k);
  for (int i = tid; i < kWarps * kMaxExperts; i += kThreads) (&wcnt[0][0])[i] = 0;
  __syncthreads();

  // ---- stable ranks within the CTA and the CTA's histogram (pairs in order)
  const int np = tb * k;  // <= kRouteTokens * 16 = kThreads
  const int e = tid < np ? sel[tid] : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(peers);
  __syncthreads();
  if (e >= 0) {
    int r = rank;
    for (int w = 0; w < warp; ++w) r += wcnt[w][e];
    ws.rank_cta[tok0 * k + tid] = r;
  }
  for (int x2 = tid; x2 < E; x2 += kThreads) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) c += wcnt[w][x2];
    ws.hist[(size_t)x2 * gridDim.x + blockIdx.x] = c;
  }

  // ---- the last CTA to finish builds the slot layout for the whole batch
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int ticket = atomicAdd(ws.meta + kMetaDone, 1);
    is_last = (ticket == (int)gridDim.x - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  route_finish(dm, ws, gridDim.x);
}

// One warp copies a row of nv 16-byte vectors with each lane's loads in
// flight together (a row of d = 4096 bf16 is one batch of 16 vectors per
// lane), instead of one load-store round trip per vector.
__device__ __forceinline__ void copy_row(uint4* dst, const uint4* src, int nv, int lane) {
  constexpr int kV = 16;
  for (int base = 0; base < nv; base += 32 * kV) {
    uint4 r[kV];
#pragma unroll
    for (int i = 0; i < kV; ++i) {
      const int j = base + lane + 32 * i;
      if (j < nv) r[i] = __ldg(src + j);
    }
#pragma unroll
    for (int i = 0; i < kV; ++i) {
      const int j = base + lane + 32 * i;
      if (j < nv) dst[j] = r[i];
    }
  }
}

template <typename TX>
__global__ void __launch_bounds__(256) permute_kernel(Dims dm, Workspace ws, const TX* x,
                                                      int tpc) {
  grid_dep_wait();
  const int item = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int k = dm.k, E = dm.E, P = dm.T * dm.k;
  const int n_cta = (dm.T + tpc - 1) / tpc;
  constexpr int kVec = 16 / sizeof(TX);
  const int nv = dm.d / kVec;
  const int nz = dm.d / 4;  // float4 per Y row
  if (item < P) {
    const int t = item / k;
    const int e = __ldcg(ws.topk_idx + item);
    const int cta = t / tpc;
    if (!moe_in_bounds(ws.status, e >= 0 && e < E)) return;
    const int slot = __ldcg(ws.expert_off + e) + __ldcg(ws.hist + (size_t)e * n_cta + cta) +
                     __ldcg(ws.rank_cta + item);
    if (!moe_in_bounds(ws.status, slot >= 0 && slot < dm.slots_routed)) return;
    if (lane == 0) {
      ws.perm[slot] = t;
      ws.slot_of[item] = slot;
      ws.slot_w[slot] = __ldcg(ws.topk_w + item);
    }
    uint4* dst = reinterpret_cast<uint4*>(static_cast<TX*>(ws.xperm) + (size_t)slot * dm.d);
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * dm.d);
    copy_row(dst, src, nv, lane);
    if (!dm.direct_combine && __ldcg(ws.y_zero + e)) {  // the GEMV path adds split partials into Y
      float4* yz = reinterpret_cast<float4*>(ws.y + (size_t)slot * dm.d);
      for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else if (item < P + E) {
    // padding slots: marked in perm; their X_perm rows are left as they are
    // (every kernel masks the columns of tokens past a group's count)
    const int e = item - P;
    const int s0 = __ldcg(ws.expert_off + e) + __ldcg(ws.expert_cnt + e);
    const int s1 = __ldcg(ws.expert_off + e + 1);
    for (int s = s0 + lane; s < s1; s += 32) ws.perm[s] = -1;
  } else if (item < P + E + dm.S * dm.T) {
    if (dm.direct_combine || !__ldcg(ws.y_zero + E)) return;
    const int q = item - P - E;
    const int sh = q / dm.T, t = q % dm.T;
    float4* yz =
        reinterpret_cast<float4*>(ws.y + (size_t)(dm.slots_routed + sh * dm.T_pad + t) * dm.d);
    for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else if (dm.direct_combine && item < P + E + dm.S * dm.T + dm.T) {
    // direct combine: the output accumulator rows Y[0..T) start at zero
    const int t = item - P - E - dm.S * dm.T;
    float4* yz = reinterpret_cast<float4*>(ws.y + (size_t)t * dm.d);
    for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Small batches (T <= kSmallTokens): the whole routing step in one CTA of
// 16 warps with no cross-CTA ticket and three CTA barriers: logits (every
// warp), top-k (a warp per token), the layout (warp 0, small_layout), then
// the permute copies of the x rows and the zeroing of the Y rows that the
// row stream adds into.
constexpr int kSmallThreads = 512;
constexpr int kSmallWarps = kSmallThreads / 32;

// Shared memory of the small-batch layout.
struct SmallLayout {
  int cnt[kMaxExperts];       // pairs per expert
  int gidx[kMaxExperts];      // group (= 8-slot block) of each touched expert
  int gpath[kMaxExperts + 8]; // path of each group (routed, then shared)
  int yzero[kMaxExperts + 1]; // 1: the expert's Y rows start at zero (last: shared)
};

// The layout of a batch of T <= kSmallTokens tokens, by one warp. Every
// touched expert holds at most 4 pairs, so it is one group in one block of
// kSlotAlign slots, in expert order; each shared expert is one group of T
// tokens. Writes the same records as build_layout (groups, paths, lists,
// cleared union counts, meta, counters) and each pair's slot (slot_s; perm,
// slot_of, slot_w, padding marks). cnt[] must be zero on entry.
__device__ void small_layout(const Dims& dm, const Workspace& ws, const int* sel,
                             const float* selw, int* slot_s, SmallLayout& L, int lane) {
  const int E = dm.E, T = dm.T, k = dm.k, S = dm.S, P = T * k;
  const unsigned lt = (1u << lane) - 1u;
  for (int p = lane; p < P; p += 32) atomicAdd(&L.cnt[sel[p]], 1);
  __syncwarp();
  // groups on the all-rows tensor-core path by size, for the join rule
  int n_tc_size = 0, n_grp = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    const int c = e < E ? L.cnt[e] : 0;
    n_grp += __popc(__ballot_sync(0xffffffffu, c > 0));
    n_tc_size += __popc(__ballot_sync(0xffffffffu, c > 0 && group_path_of(dm, c) == kPathTcAll));
  }
  n_grp += S;
  n_tc_size += group_path_of(dm, T) == kPathTcAll ? S : 0;
  const bool join = tc_join(dm, n_tc_size, n_grp);
  // touched experts in expert order: group index and path
  int n_touched = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    const int c = e < E ? L.cnt[e] : 0;
    const unsigned bal = __ballot_sync(0xffffffffu, c > 0);
    if (c > 0) {
      const int g = n_touched + __popc(bal & lt);
      const int path = joined_path(group_path_of(dm, c), join);
      L.gidx[e] = g;
      L.gpath[g] = path;
      Group gr;
      gr.expert = e;
      gr.slot0 = g * kSlotAlign;
      gr.m = c;
      gr.xrow0 = g * kSlotAlign;
      ws.groups[g] = gr;
      ws.group_path[g] = path;
      ws.union_cnt[g] = 0;
      // padding slots of the block: marked in perm (their X_perm rows are
      // never used: every kernel masks the columns past a group's count)
      for (int r = c; r < kSlotAlign; ++r) ws.perm[g * kSlotAlign + r] = -1;
    }
    if (e < E) L.yzero[e] = c > 0 && adds_into_y(joined_path(group_path_of(dm, c), join));
    n_touched += __popc(bal);
  }
  const int n_groups = n_touched + S;
  if (lane < S) {  // shared experts: one group of all T tokens each
    const int g = n_touched + lane;
    const int path = joined_path(group_path_of(dm, T), join);
    L.gpath[g] = path;
    Group gr;
    gr.expert = E + lane;
    gr.slot0 = dm.slots_routed + lane * dm.T_pad;
    gr.m = T;
    gr.xrow0 = 0;
    ws.groups[g] = gr;
    ws.group_path[g] = path;
    ws.union_cnt[g] = 0;
  }
  __syncwarp();
  // GEMV and tensor-core lists in group order (a candidate is on both)
  int n_gv = 0, n_tc = 0, n_cand = 0, n_tc_sh = 0, any_gv_sh = 0, n_fz = 0;
  for (int g0 = 0; g0 < n_groups; g0 += 32) {
    const int g = g0 + lane;
    const int path = g < n_groups ? L.gpath[g] : kPathNone;
    const bool gv = g < n_groups && on_gemv_list(path);
    const bool tc = g < n_groups && on_tc_list(path);
    const bool cand = g < n_groups && path == kPathCand;
    const unsigned bgv = __ballot_sync(0xffffffffu, gv), btc = __ballot_sync(0xffffffffu, tc);
    if (gv) ws.gemv_list[n_gv + __popc(bgv & lt)] = g;
    if (tc) ws.tc_list[n_tc + __popc(btc & lt)] = g;
    n_gv += __popc(bgv);
    n_tc += __popc(btc);
    n_cand += __popc(__ballot_sync(0xffffffffu, cand));
    n_tc_sh += __popc(__ballot_sync(0xffffffffu, tc && !cand && g >= n_touched));
    n_fz += __popc(__ballot_sync(0xffffffffu, g < n_groups && path == kPathFused));
    any_gv_sh |= __ballot_sync(0xffffffffu, g < n_groups && adds_into_y(path) && g >= n_touched) != 0u;
  }
  if (lane == 0) L.yzero[E] = any_gv_sh;
  // each pair's slot: its expert's block + its rank among the expert's pairs
  for (int p = lane; p < P; p += 32) {
    const int e = sel[p];
    int r = 0;
    for (int q = 0; q < p; ++q) r += sel[q] == e;
    int slot = L.gidx[e] * kSlotAlign + r;
    if (!moe_in_bounds(ws.status, slot >= 0 && slot < dm.slots_routed)) slot = 0;
    slot_s[p] = slot;
    ws.perm[slot] = p / k;
    ws.slot_of[p] = slot;
    ws.slot_w[slot] = selw[p];
  }
  if (lane < kCntWords) {
    unsigned long long v = 0ull;
    if (lane == kCntGemv) v = n_gv - n_cand + n_fz;  // candidates: counted by the kernel that takes them
    if (lane == kCntTc) v = n_tc - n_cand;
    if (lane == kCntDownRows && dm.mode != kModeTc)  // the GEMV kernel adds its rows
      v = (unsigned long long)(n_tc - n_cand - n_tc_sh) * dm.F +
          (unsigned long long)n_tc_sh * dm.Fs;
    if (lane == kCntRoutedH) v = (unsigned long long)P * dm.F;
    if (lane == kCntSharedH) v = (unsigned long long)S * T * dm.Fs;
    ws.counters[lane] = v;
  }
  if (lane == 0) {
    ws.meta[kMetaRoutedGroups] = n_touched;
    ws.meta[kMetaGroups] = n_groups;
    ws.meta[kMetaSlotsUsed] = n_touched * kSlotAlign;
    ws.meta[kMetaExpertsTouched] = n_touched;
    ws.meta[kMetaGemvCount] = n_gv;
    ws.meta[kMetaTcCount] = n_tc;
    ws.meta[kMetaDone] = 0;
    ws.meta[kMetaDownDone] = 0;
    ws.meta[kMetaTcQueue] = 0;
  }
  __syncwarp();
}

template <typename TX>
__global__ void __launch_bounds__(kSmallThreads, 1)
    route_small_kernel(Dims dm, Workspace ws, const TX* x, const TX* Wr, const float* bias) {
  __shared__ float lg[kSmallTokens][kMaxExperts + 1];
  __shared__ float lpart[4][kSmallTokens][kMaxExperts];  // split-d partial logits
  __shared__ int sel[kSmallTokens * 16];
  __shared__ float selw[kSmallTokens * 16];
  __shared__ int slot_s[kSmallTokens * 16];
  __shared__ SmallLayout L;

  grid_dep_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = dm.E, d = dm.d, T = dm.T, k = dm.k;
  const int P = T * k;

  // (token, expert) dots; with fewer dots than warps each is split into ns
  // slices of d (slices added in order), so every warp has one
  const int TE = T * E;
  const int ns = TE * 4 <= kSmallWarps ? 4 : TE * 2 <= kSmallWarps ? 2 : 1;
  const int dsl = d / ns;  // d is a multiple of 256: slices stay whole vectors
  for (int task = warp; task < TE * ns; task += kSmallWarps) {
    const int sl = task / TE, te = task % TE;
    const int t = te / E, e = te % E;
    const float a = row_dot<TX>(x + (size_t)t * d + (size_t)sl * dsl,
                                Wr + (size_t)e * d + (size_t)sl * dsl, dsl, lane);
    if (lane == 0) lpart[sl][t][e] = a;
  }
  for (int e = tid; e < E; e += kSmallThreads) L.cnt[e] = 0;
  __syncthreads();
  if (warp < T) {  // warp t: token t's logits (slices in order, + bias) and top-k
    for (int e = lane; e < E; e += 32) {
      float a = 0.f;
      for (int sl = 0; sl < ns; ++sl) a += lpart[sl][warp][e];
      lg[warp][e] = a + (bias ? bias[e] : 0.f);
    }
    __syncwarp();
    topk_token(dm, ws, lg[warp], warp, lane, sel + warp * k, selw + warp * k);
  } else {  // the other warps clear the next kernels' cross-CTA tickets
    for (int x2 = tid - T * 32; x2 < dm.sk_ctas; x2 += kSmallThreads - T * 32)
      ws.sk_flags[x2] = 0;
    for (int x2 = tid - T * 32; x2 < dm.tc_part_units; x2 += kSmallThreads - T * 32)
      ws.tc_ticket[x2] = 0;
  }
  __syncthreads();
  if (warp == 0) small_layout(dm, ws, sel, selw, slot_s, L, lane);
  __syncthreads();
  // copies: one warp per pair (x row to X_perm; the Y rows the row stream
  // adds into start at zero), then the shared experts' Y rows
  constexpr int kVec = 16 / sizeof(TX);
  const int nv = d / kVec, nz = d / 4;
  for (int p = warp; p < P; p += kSmallWarps) {
    const int slot = slot_s[p];
    uint4* dst = reinterpret_cast<uint4*>(static_cast<TX*>(ws.xperm) + (size_t)slot * d);
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(p / k) * d);
    copy_row(dst, src, nv, lane);
    if (!dm.direct_combine && L.yzero[sel[p]]) {
      float4* yz = reinterpret_cast<float4*>(ws.y + (size_t)slot * d);
      for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  if (dm.direct_combine) {  // the output accumulator rows Y[0..T) start at zero
    for (int t = warp; t < T; t += kSmallWarps) {
      float4* yz = reinterpret_cast<float4*>(ws.y + (size_t)t * d);
      for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else if (L.yzero[E]) {
    for (int q = warp; q < dm.S * T; q += kSmallWarps) {
      const int sh = q / T, t = q % T;
      float4* yz = reinterpret_cast<float4*>(ws.y + (size_t)(dm.slots_routed + sh * dm.T_pad + t) * d);
      for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

}  // namespace

// Tokens per router CTA: few at decode so that the batch spreads over many
// SMs, more at prefill to keep the per-CTA histograms short; the staged rows
// stay within kStageBytes so that two router CTAs fit on an SM.
constexpr size_t kStageBytes = 80 * 1024;

int route_tokens_per_cta(const Dims& dm, int elem_bytes) {
  if (dm.T <= 256) return 2;
  int tpc = kRouteTokens;
  while (tpc > 2 && (size_t)tpc * dm.d * elem_bytes > kStageBytes) tpc >>= 1;
  return tpc;
}

bool route_is_small(const Dims& dm) { return dm.T <= kSmallTokens; }

namespace {

template <typename TX, int TPC>
cudaError_t launch_route_t(const Dims& dm, const Workspace& ws, const TX* x, const TX* Wr,
                           const float* bias, int tpc, cudaStream_t st) {
  const int grid = (dm.T + tpc - 1) / tpc;
  const size_t xbytes = (size_t)tpc * dm.d * sizeof(TX);
  const int stage_x = xbytes <= kStageBytes;
  const cudaError_t e = smem_limit(route_kernel<TX, TPC>, (int)kStageBytes);
  if (e != cudaSuccess) return e;
  return launch_k(route_kernel<TX, TPC>, grid, kThreads, stage_x ? xbytes : 0, st, dm, ws, x,
                  Wr, bias, tpc, stage_x);
}

template <typename TX>
cudaError_t launch_route_x(const Dims& dm, const Workspace& ws, const TX* x, const TX* Wr,
                           const float* bias, cudaStream_t st) {
  const int tpc = route_tokens_per_cta(dm, sizeof(TX));
  switch (tpc) {
    case 2: return launch_route_t<TX, 2>(dm, ws, x, Wr, bias, tpc, st);
    case 4: return launch_route_t<TX, 4>(dm, ws, x, Wr, bias, tpc, st);
    case 8: return launch_route_t<TX, 8>(dm, ws, x, Wr, bias, tpc, st);
    default: return launch_route_t<TX, kRouteTokens>(dm, ws, x, Wr, bias, tpc, st);
  }
}

}  // namespace

cudaError_t launch_route(const Dims& dm, const Workspace& ws, const void* x, const void* Wr,
                         const float* bias, bool bf16, cudaStream_t st) {
  if (route_is_small(dm)) {
    if (bf16)
      return launch_k(route_small_kernel<__nv_bfloat16>, 1, kSmallThreads, 0, st, dm, ws,
                      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wr),
                      bias);
    return launch_k(route_small_kernel<float>, 1, kSmallThreads, 0, st, dm, ws,
                    static_cast<const float*>(x), static_cast<const float*>(Wr), bias);
  }
  if (bf16)
    return launch_route_x(dm, ws, static_cast<const __nv_bfloat16*>(x),
                          static_cast<const __nv_bfloat16*>(Wr), bias, st);
  return launch_route_x(dm, ws, static_cast<const float*>(x), static_cast<const float*>(Wr), bias,
                        st);
}

cudaError_t launch_permute(const Dims& dm, const Workspace& ws, const void* x, bool bf16,
                           cudaStream_t st) {
  const int items = dm.T * dm.k + dm.E + dm.S * dm.T + (dm.direct_combine ? dm.T : 0);
  const int grid = (items + 7) / 8;
  const int tpc = route_tokens_per_cta(dm, bf16 ? 2 : 4);
  if (bf16)
    return launch_k(permute_kernel<__nv_bfloat16>, grid, 256, 0, st, dm, ws,
                    static_cast<const __nv_bfloat16*>(x), tpc);
  return launch_k(permute_kernel<float>, grid, 256, 0, st, dm, ws, static_cast<const float*>(x),
                  tpc);
}

}  // namespace moe
