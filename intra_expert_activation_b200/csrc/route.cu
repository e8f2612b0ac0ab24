// Router: logits, softmax over all experts, top-k (+ renormalisation), and a
// deterministic stable counting sort of the routed (token, expert) pairs into
// per-expert slot ranges and expert token groups. The pages keep the dense
// model's router as it is [gist.science EN "Uncovering Intra-expert
// Activation Sparsity for Efficient Mixture-of-Expert Model Execution",
// Technical Summary > Methodology > System Implementation in vLLM].
//
// route_kernel, one CTA per `tpc` tokens (2 at decode, kRouteTokens at
// prefill):
//   logits   warp tasks (token, expert): the lanes stride d with batches of
//            16-byte loads of the x row and the W_router row and reduce with
//            a butterfly (fp32, a fixed summation order);
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
//   zero the padding slots.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxExperts = 256;
constexpr int kSmallTokens = 4;  // single-CTA routing (and permute) up to this batch

// Total order used by the top-k: larger logit first, then lower index.
__device__ __forceinline__ bool better(float va, int ea, float vb, int eb) {
  return va > vb || (va == vb && ea < eb);
}

template <typename TX>
struct XVec;
template <>
struct XVec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load_shared(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(b[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ static void load(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
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
struct XVec<float> {
  static constexpr int N = 4;
  __device__ static void load_shared(const float* p, float (&f)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
  __device__ static void load(const float* p, float (&f)[4]) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
};

// Path of a group from its token count and the requested mode (the
// batch-size switch of the pages, taken per expert token group).
__device__ __forceinline__ int group_path_of(const Dims& dm, int m) {
  if (dm.no_tc || dm.mode == kModeGemv) return kPathGemv;
  if (dm.mode == kModeTc) return kPathTcAll;  // gathered or not: decided by the union scan
  if (dm.mode == kModeTcAll) return kPathTcAll;
  return m <= dm.gemv_max ? kPathGemv : kPathTcAll;  // auto and dense
}

// Last CTA: histograms -> base offsets, expert slot ranges, token groups, the
// path of every group, the GEMV work items. s_a / s_b are free shared
// scratch of at least 2 * kListMax + 1 and kListMax ints.
__device__ void build_layout(const Dims& dm, const Workspace& ws, const int* cnt, int* poff,
                             int* s_a, int* s_b);

__device__ void route_finish(const Dims& dm, const Workspace& ws, int n_cta, int* s_a,
                             int* s_b) {
  __shared__ int cnt[kMaxExperts];
  __shared__ int poff[kMaxExperts + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = dm.E;
  // per expert: exclusive scan of its CTA counts (contiguous, expert-major);
  // each lane takes 8 consecutive CTAs of a 256-CTA chunk, so a chunk is one
  // load round trip
  for (int e = warp; e < E; e += blockDim.x / 32) {
    int* h = ws.hist + static_cast<size_t>(e) * n_cta;
    int carry = 0;
    for (int c0 = 0; c0 < n_cta; c0 += 256) {
      int v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = c0 + lane * 8 + i;
        v[i] = c < n_cta ? __ldcg(h + c) : 0;
      }
      int sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) sum += v[i];
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      int run = carry + incl - sum;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = c0 + lane * 8 + i;
        if (c < n_cta) h[c] = run;
        run += v[i];
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) cnt[e] = carry;
  }
  if (tid < kCntWords) ws.counters[tid] = 0ull;
  __syncthreads();
  build_layout(dm, ws, cnt, poff, s_a, s_b);
}

// From the per-expert pair counts cnt[E] (shared memory): expert slot ranges
// poff[E+1] (shared), token groups, the path of every group, the GEMV work
// items, counters and meta. s_a / s_b: shared scratch of 2 * kListMax + 1 and
// kListMax ints. Called by every thread of the CTA; counters must be zero.
__device__ void build_layout(const Dims& dm, const Workspace& ws, const int* cnt, int* poff,
                             int* s_a, int* s_b) {
  __shared__ int n_gemv_s, n_items_s;
  const int tid = threadIdx.x;
  const int E = dm.E, T = dm.T, k = dm.k;
  const int mt = dm.no_tc ? 8 : kGemvTokens;
  int* gemv_g = s_a;                  // [kListMax] GEMV groups in group order
  int* item_off = s_a + kListMax;     // [kListMax + 1]
  int* splits = s_b;                  // [kListMax]
  if (tid == 0) {
    int touched = 0;
    poff[0] = 0;
    for (int x = 0; x < E; ++x) {
      const int me = cnt[x];
      touched += me > 0;
      poff[x + 1] = poff[x] + (me + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
    }
    int ng = 0, n_gemv = 0, n_tc = 0, units = 0;
    unsigned long long tc_rows = 0;
    auto add_group = [&](int expert, int slot0, int m, int xrow0, int F_e) {
      if (ng >= dm.groups_max) return;
      Group gr;
      gr.expert = expert;
      gr.slot0 = slot0;
      gr.m = m;
      gr.xrow0 = xrow0;
      ws.groups[ng] = gr;
      const int path = group_path_of(dm, m);
      ws.group_path[ng] = path;
      if (path == kPathGemv) {
        gemv_g[n_gemv] = ng;
        ws.gemv_list[n_gemv++] = ng;
        units += (m + mt - 1) / mt;
      } else {
        ws.tc_list[n_tc++] = ng;
        tc_rows += F_e;
      }
      ++ng;
    };
    for (int x = 0; x < E; ++x) {
      const int me = cnt[x];
      int zero = 0;
      if (me > 0) {
        const int n_g = (me + kGroupMax - 1) / kGroupMax;
        int gsz = (me + n_g - 1) / n_g;
        gsz = (gsz + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
        for (int g = 0; g * gsz < me; ++g) {
          const int m = min(gsz, me - g * gsz);
          zero |= group_path_of(dm, m) == kPathGemv;
          add_group(x, poff[x] + g * gsz, m, poff[x] + g * gsz, dm.F);
        }
      }
      ws.y_zero[x] = zero;
    }
    ws.meta[kMetaRoutedGroups] = ng;
    int zero_s = 0;
    for (int sh = 0; sh < dm.S; ++sh) {
      const int n_g = (T + kGroupMax - 1) / kGroupMax;
      int gsz = (T + n_g - 1) / n_g;
      gsz = (gsz + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
      for (int g = 0; g * gsz < T; ++g) {
        const int m = min(gsz, T - g * gsz);
        zero_s |= group_path_of(dm, m) == kPathGemv;
        add_group(E + sh, dm.slots_routed + sh * dm.T_pad + g * gsz, m, g * gsz, dm.Fs);
      }
    }
    ws.y_zero[E] = zero_s;
    // GEMV items: every unit (group, pass of mt tokens) of group i is cut into
    // splits[i] neuron ranges of whole bitmap words, about three items per SM
    // (the GEMV kernel balances them with a queue)
    const int target = max(1, 3 * dm.n_sms / max(units, 1));
    int items = 0;
    for (int i = 0; i < n_gemv; ++i) {
      const Group gr = ws.groups[gemv_g[i]];
      const int words = (gr.expert >= E ? dm.Fs : dm.F) / 32;
      const int s_min = (words + kGemvWordsMax - 1) / kGemvWordsMax;
      splits[i] = min(max(target, s_min), words);
      item_off[i] = items;
      items += (gr.m + mt - 1) / mt * splits[i];
    }
    item_off[n_gemv] = items;
    items = min(items, dm.gemv_items_max);
    n_gemv_s = n_gemv;
    n_items_s = items;
    ws.meta[kMetaGroups] = ng;
    ws.meta[kMetaSlotsUsed] = poff[E];
    ws.meta[kMetaExpertsTouched] = touched;
    ws.meta[kMetaGemvCount] = n_gemv;
    ws.meta[kMetaTcCount] = n_tc;
    ws.meta[kMetaGemvItems] = items;
    ws.meta[kMetaGemvNext] = 0;
    ws.counters[kCntGemv] = n_gemv;
    ws.counters[kCntTc] = n_tc;
    if (dm.mode != kModeTc) ws.counters[kCntDownRows] = tc_rows;  // GEMV items add theirs
    ws.counters[kCntRoutedH] = (unsigned long long)T * k * (unsigned long long)dm.F;
    ws.counters[kCntSharedH] =
        (unsigned long long)dm.S * (unsigned long long)T * (unsigned long long)dm.Fs;
    ws.meta[kMetaDone] = 0;  // ticket counter for the next forward
  }
  __syncthreads();
  for (int x = tid; x <= E; x += blockDim.x) ws.expert_off[x] = poff[x];
  for (int x = tid; x < E; x += blockDim.x) ws.expert_cnt[x] = cnt[x];
  // item descriptors: everything a GEMV CTA needs in one load
  const int n_gemv = n_gemv_s, n_items = n_items_s;
  for (int it = tid; it < n_items; it += blockDim.x) {
    int lo_i = 0, hi_i = n_gemv;
    while (hi_i - lo_i > 1) {
      const int mid = (lo_i + hi_i) >> 1;
      if (item_off[mid] <= it) lo_i = mid; else hi_i = mid;
    }
    const int g = gemv_g[lo_i];
    const Group gr = ws.groups[g];
    const int words = (gr.expert >= E ? dm.Fs : dm.F) / 32;
    const int sp = splits[lo_i];
    const int local = it - item_off[lo_i];
    const int split = local % sp, pass = local / sp;
    GemvItem d;
    d.g = g;
    d.expert = gr.expert;
    d.slot = gr.slot0 + pass * mt;
    d.mt = min(mt, gr.m - pass * mt);
    d.w0 = split * words / sp;
    d.w1 = (split + 1) * words / sp;
    d.whole = sp == 1;
    d.pad = 0;
    ws.gemv_items[it] = d;
  }
}

// Dot product of one token row with one router row, lanes over d in chunks
// of 32 x VEC elements, loads issued in batches of kBatch chunks.
template <typename TX>
__device__ __forceinline__ float row_dot(const TX* a, const TX* b, int d, int lane) {
  constexpr int VEC = XVec<TX>::N;
  constexpr int kBatch = 8;
  float acc = 0.f;
  for (int c0 = lane * VEC; c0 < d; c0 += 32 * VEC * kBatch) {
    float av[kBatch][VEC], bv[kBatch][VEC];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int c = c0 + i * 32 * VEC;
      if (c < d) {
        XVec<TX>::load(a + c, av[i]);
        XVec<TX>::load(b + c, bv[i]);
      } else {
#pragma unroll
        for (int v = 0; v < VEC; ++v) av[i][v] = bv[i][v] = 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i)
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc = fmaf(av[i][v], bv[i][v], acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// Top-k of one token's logits (one warp): the k largest, equal logits to the
// lower expert index; softmax over all experts; weights p / sum(p_sel) or p.
// Writes topk_idx / topk_w of token `tok` and the chosen experts to sel[0..k).
__device__ __forceinline__ void topk_token(const Dims& dm, const Workspace& ws, const float* lgt,
                                           int tok, int lane, int* sel) {
  const int E = dm.E, k = dm.k;
  float v[kMaxExperts / 32];
#pragma unroll
  for (int j = 0; j < kMaxExperts / 32; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < E ? lgt[e] : -INFINITY;
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
    sel[lane] = my_e;
  }
}

template <typename TX>
__global__ void __launch_bounds__(kThreads) route_kernel(Dims dm, Workspace ws, const TX* x,
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
    // ---- logits with the CTA's x rows in shared memory: a warp owns an
    // expert and all of the CTA's tokens, so one W_router load feeds tb tokens
    extern __shared__ __align__(16) uint8_t xs_raw[];
    float* xs = reinterpret_cast<float*>(xs_raw);  // [tb][d] as fp32
    constexpr int VEC = XVec<TX>::N;
    const int nvec = tb * d / VEC;
    for (int i = tid; i < nvec; i += kThreads) {
      float v[VEC];
      XVec<TX>::load(x + (size_t)tok0 * d + (size_t)i * VEC, v);
#pragma unroll
      for (int q = 0; q < VEC; q += 4)
        *reinterpret_cast<float4*>(xs + (size_t)i * VEC + q) = make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
    }
    __syncthreads();
    for (int e = warp; e < E; e += kWarps) {
      float acc[kRouteTokens];
#pragma unroll
      for (int t = 0; t < kRouteTokens; ++t) acc[t] = 0.f;
      const TX* wr = Wr + (size_t)e * d;
      for (int c = lane * VEC; c < d; c += 32 * VEC) {
        float w[VEC];
        XVec<TX>::load(wr + c, w);
#pragma unroll
        for (int t = 0; t < kRouteTokens; ++t) {
          if (t < tb) {
            const float* xr = xs + (size_t)t * d + c;
#pragma unroll
            for (int v = 0; v < VEC; v += 4) {
              const float4 xv = *reinterpret_cast<const float4*>(xr + v);
              acc[t] = fmaf(xv.x, w[v], acc[t]);
              acc[t] = fmaf(xv.y, w[v + 1], acc[t]);
              acc[t] = fmaf(xv.z, w[v + 2], acc[t]);
              acc[t] = fmaf(xv.w, w[v + 3], acc[t]);
            }
          }
        }
      }
      const float b = bias ? bias[e] : 0.f;
#pragma unroll
      for (int t = 0; t < kRouteTokens; ++t) {
        if (t < tb) {
          float a = acc[t];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
          if (lane == 0) lg[t][e] = a + b;
        }
      }
    }
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
  static_assert(sizeof(lg) >= sizeof(int) * (2 * kListMax + 1), "finish scratch");
  static_assert(sizeof(wcnt) >= sizeof(int) * kListMax, "finish scratch");
  route_finish(dm, ws, gridDim.x, reinterpret_cast<int*>(&lg[0][0]), &wcnt[0][0]);
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
    const int slot = __ldcg(ws.expert_off + e) + __ldcg(ws.hist + (size_t)e * n_cta + cta) +
                     __ldcg(ws.rank_cta + item);
    if (lane == 0) {
      ws.perm[slot] = t;
      ws.slot_of[item] = slot;
    }
    uint4* dst = reinterpret_cast<uint4*>(static_cast<TX*>(ws.xperm) + (size_t)slot * dm.d);
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * dm.d);
    for (int i = lane; i < nv; i += 32) dst[i] = __ldg(src + i);
    if (__ldcg(ws.y_zero + e)) {  // the GEMV path adds split partials into Y
      float4* yz = reinterpret_cast<float4*>(ws.y + (size_t)slot * dm.d);
      for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else if (item < P + E) {
    const int e = item - P;
    const int s0 = __ldcg(ws.expert_off + e) + __ldcg(ws.expert_cnt + e);
    const int s1 = __ldcg(ws.expert_off + e + 1);
    for (int s = s0; s < s1; ++s) {
      if (lane == 0) ws.perm[s] = -1;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<TX*>(ws.xperm) + (size_t)s * dm.d);
      for (int i = lane; i < nv; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
    }
  } else if (item < P + E + dm.S * dm.T) {
    if (!__ldcg(ws.y_zero + E)) return;
    const int q = item - P - E;
    const int sh = q / dm.T, t = q % dm.T;
    float4* yz =
        reinterpret_cast<float4*>(ws.y + (size_t)(dm.slots_routed + sh * dm.T_pad + t) * dm.d);
    for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Small batches (T <= kSmallTokens): the whole routing step in one CTA of
// 32 warps with no cross-CTA ticket: logits, top-k, in-order stable ranks,
// layout, and the permute copies of the x rows (and zeroing of the Y rows
// that GEMV splits add into).
constexpr int kSmallThreads = 512;
constexpr int kSmallWarps = kSmallThreads / 32;

template <typename TX>
__global__ void __launch_bounds__(kSmallThreads, 1)
    route_small_kernel(Dims dm, Workspace ws, const TX* x, const TX* Wr, const float* bias) {
  __shared__ float lg[kSmallTokens][kMaxExperts + 1];
  __shared__ int sel[kSmallTokens * 16];
  __shared__ int slot_s[kSmallTokens * 16];
  __shared__ int cnt[kMaxExperts];
  __shared__ int poff[kMaxExperts + 1];
  __shared__ int scratch_a[2 * kListMax + 1];
  __shared__ int scratch_b[kListMax];

  grid_dep_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = dm.E, d = dm.d, T = dm.T, k = dm.k;
  const int P = T * k;

  for (int task = warp; task < T * E; task += kSmallWarps) {
    const int t = task / E, e = task % E;
    const float a = row_dot<TX>(x + (size_t)t * d, Wr + (size_t)e * d, d, lane);
    if (lane == 0) lg[t][e] = a + (bias ? bias[e] : 0.f);
  }
  for (int e = tid; e < E; e += kSmallThreads) cnt[e] = 0;
  if (tid < kCntWords) ws.counters[tid] = 0ull;
  __syncthreads();
  for (int t = warp; t < T; t += kSmallWarps)
    topk_token(dm, ws, lg[t], t, lane, sel + t * k);
  __syncthreads();
  // stable rank of pair p among earlier pairs of the same expert
  for (int p = tid; p < P; p += kSmallThreads) {
    const int e = sel[p];
    int r = 0;
    for (int q = 0; q < p; ++q) r += sel[q] == e;
    slot_s[p] = r;
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  build_layout(dm, ws, cnt, poff, scratch_a, scratch_b);
  __syncthreads();
  for (int p = tid; p < P; p += kSmallThreads) {
    const int slot = poff[sel[p]] + slot_s[p];
    slot_s[p] = slot;
    ws.perm[slot] = p / k;
    ws.slot_of[p] = slot;
  }
  __syncthreads();
  // copies: one warp per pair, then padding slots, then shared Y rows
  constexpr int kVec = 16 / sizeof(TX);
  const int nv = d / kVec, nz = d / 4;
  for (int p = warp; p < P; p += kSmallWarps) {
    const int slot = slot_s[p];
    uint4* dst = reinterpret_cast<uint4*>(static_cast<TX*>(ws.xperm) + (size_t)slot * d);
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(p / k) * d);
    for (int i = lane; i < nv; i += 32) dst[i] = __ldg(src + i);
    if (ws.y_zero[sel[p]]) {
      float4* yz = reinterpret_cast<float4*>(ws.y + (size_t)slot * d);
      for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  for (int e = warp; e < E; e += kSmallWarps) {
    for (int sl = poff[e] + cnt[e]; sl < poff[e + 1]; ++sl) {
      if (lane == 0) ws.perm[sl] = -1;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<TX*>(ws.xperm) + (size_t)sl * d);
      for (int i = lane; i < nv; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
    }
  }
  if (ws.y_zero[E]) {
    for (int q = warp; q < dm.S * T; q += kSmallWarps) {
      const int sh = q / T, t = q % T;
      float4* yz = reinterpret_cast<float4*>(ws.y + (size_t)(dm.slots_routed + sh * dm.T_pad + t) * d);
      for (int i = lane; i < nz; i += 32) yz[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

}  // namespace

// Tokens per router CTA: few at decode so that the (token, expert) dot
// products spread over many SMs, more at prefill to keep the per-CTA
// histograms short.
int route_tokens_per_cta(const Dims& dm) {
  if (dm.T <= 256) return 2;
  int tpc = kRouteTokens;  // rows staged as fp32 in shared memory: at most 192 KB
  while (tpc > 2 && (size_t)tpc * dm.d * 4 > 192 * 1024) tpc >>= 1;
  return tpc;
}

bool route_is_small(const Dims& dm) { return dm.T <= kSmallTokens; }

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
  const int tpc = route_tokens_per_cta(dm);
  const int grid = (dm.T + tpc - 1) / tpc;
  // with 16 tokens per CTA, stage their rows in shared memory when they fit
  const size_t xbytes = (size_t)tpc * dm.d * 4;
  const int stage_x = tpc > 2 && xbytes <= 192 * 1024;
  const size_t smem = stage_x ? xbytes : 0;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 192 * 1024);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(route_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               192 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (bf16)
    return launch_k(route_kernel<__nv_bfloat16>, grid, kThreads, smem, st, dm, ws,
                    static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wr),
                    bias, tpc, stage_x);
  return launch_k(route_kernel<float>, grid, kThreads, smem, st, dm, ws,
                  static_cast<const float*>(x), static_cast<const float*>(Wr), bias, tpc,
                  stage_x);
}

cudaError_t launch_permute(const Dims& dm, const Workspace& ws, const void* x, bool bf16,
                           cudaStream_t st) {
  const int items = dm.T * dm.k + dm.E + dm.S * dm.T;
  const int grid = (items + 7) / 8;
  const int tpc = route_tokens_per_cta(dm);
  if (bf16)
    return launch_k(permute_kernel<__nv_bfloat16>, grid, 256, 0, st, dm, ws,
                    static_cast<const __nv_bfloat16*>(x), tpc);
  return launch_k(permute_kernel<float>, grid, 256, 0, st, dm, ws, static_cast<const float*>(x),
                  tpc);
}

}  // namespace moe
