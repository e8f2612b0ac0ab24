// Down projection for expert token groups with few tokens (decode): stream
// only the W_down rows in the group's active-neuron union and multiply them
// by the tokens' h values.
//
// This is the low-batch side of the pages' batch-size switch [gist.science
// EN "Uncovering Intra-expert Activation Sparsity for Efficient
// Mixture-of-Expert Model Execution", Technical Summary > Methodology >
// System Implementation in vLLM > "Dynamic Switching"]: with one to a few
// tokens per expert the down projection is a matrix-vector product whose
// cost is the bytes of the rows it reads ["Fused Up-Down Projection": only
// the active neurons' weights are fetched].
//
// Work split. A unit is (GEMV group, pass of up to MT of its tokens); its
// rows are the group's union rows, whose count the gate/up epilogue left in
// union_cnt. The units' rows, in (group, pass, neuron) order, form one
// sequence of R rows; CTA c (one per SM) takes rows [R c / G, R (c+1) / G),
// so every SM streams the same number of rows, with no work queue.
//
// Inside a CTA, warp-specialised. The producer warp walks the CTA's share of
// the union bitmaps (32 words at a time it compacts the set bits into a row
// list) and fills a ring of shared-memory stages of kBatch rows: one bulk
// copy (cp.async.bulk, mbarrier completion) per row brings the row's bytes
// of the current column block (up to 4 KB), and cp.async copies of the
// tokens' h values arrive on the same barrier when they land. Each of the
// 8 consumer warps owns a 512-byte column slice of the block (with narrow d
// several warps share a slice and take alternate stages) and multiplies the
// landed rows: bf16 on the tensor cores (mma.sync m16n8k8: 16 columns x 8
// rows x up to 8 tokens, fp32 accumulation), fp32 with packed fp32x2 FMAs.
// Rows sit at a stride of the block plus 16 bytes, so the eight rows of a
// transposed 8x8 matrix load fall in eight different bank groups. When the
// unit changes a consumer adds its partial sums into Y[slot][columns]
// (zeroed by the router) with vector fp32 atomics: the partials of a unit are
// summed in arrival order, so results agree to fp32 rounding, not bitwise,
// between runs on this path.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kConsumers = 8;
constexpr int kThreads = (kConsumers + 1) * 32;  // + the producer warp
constexpr int kBatch = 8;            // rows per stage (the mma's K)
constexpr int kSliceBytes = 512;     // row bytes per consumer warp
constexpr int kBlockBytes = kConsumers * kSliceBytes;  // column block: 4 KB of a row
constexpr int kRowPad = 16;          // row stride = block bytes + 16
constexpr int kHBytes = 32;          // h bytes per row: 4 x bf16 or 8 x fp32
constexpr int kMaxStages = 6;
constexpr int kSmemBudget = 190 * 1024;  // stages; the result staging comes on top
constexpr int kListRows = 256;       // producer's row list (uint16 neuron indices)
constexpr int kTight = 4096;         // barrier probes before sleeping: stages arrive every few us
constexpr int kYStride = 260;        // floats per staged result row of a consumer warp
constexpr int kYBytes = kGemvTokens * kYStride * 4;  // a consumer warp's result staging

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// Packed pair of fp32 values and d = a * b + d on both halves.
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

// Four 8x8 bf16 matrices from shared memory, transposed (lane i supplies the
// address of row i % 8 of matrix i / 8).
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// d += A (16 x 8, bf16) * B (8 x 8, bf16), fp32 accumulation.
__device__ __forceinline__ void mma_16x8x8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// Arrive on bar once this thread's earlier cp.async copies have landed (the
// barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Bulk copy of `bytes` (a multiple of 16) from global to shared memory,
// completion counted on bar as transaction bytes.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Stage geometry for a row of row_bytes: the column block (<= 4 KB), the
// stage size and the number of stages that fit the budget.
struct Geometry {
  int block, stride, stage, n_stages;
};
__host__ __device__ inline Geometry geometry(int row_bytes) {
  Geometry g;
  g.block = row_bytes < kBlockBytes ? row_bytes : kBlockBytes;
  g.stride = g.block + kRowPad;
  g.stage = kBatch * g.stride + kBatch * kHBytes + 16;  // rows | h | meta
  g.n_stages = kSmemBudget / g.stage;
  if (g.n_stages > kMaxStages) g.n_stages = kMaxStages;
  return g;
}

// Where a CTA's share of the row sequence starts.
struct Start {
  int i;        // GEMV list index of the first group
  int p;        // pass within it
  int w;        // bitmap word of the first row
  uint32_t m;   // mask of the rows of word w that are still to come
  int rows;     // rows of this CTA
  int g, row;   // the first group and the row within its pass (prologue scratch)
};

// The producer's walk over its CTA's rows: group list index, pass, next word
// and the mask for it, rows still to produce, and the unit being produced.
struct Walk {
  int i, p, w;
  uint32_t m;
  int left;
  int n_gv;  // GEMV groups
  int g, words, passes, slot0, m_tok, expert;  // unit data of group i
  int serial;  // increments whenever the unit (group, pass) changes
};

// Loads group i's unit data; false past the end of the GEMV list.
__device__ __forceinline__ bool walk_load_group(const Dims& dm, const Workspace& ws, Walk& k,
                                                int MT) {
  if (k.i >= k.n_gv) return false;
  k.g = __ldcg(ws.gemv_list + k.i);
  const Group gr = ws.groups[k.g];
  k.expert = gr.expert;
  k.slot0 = gr.slot0;
  k.m_tok = gr.m;
  k.passes = (gr.m + MT - 1) / MT;
  k.words = (gr.expert >= dm.E ? dm.Fs : dm.F) / 32;
  return true;
}

// Next run of rows of one unit into the list: the set bits of up to 32
// bitmap words (one per lane), at most kListRows and at most k.left rows.
// Returns the number of rows (0 once the walk is over). Whole warp.
__device__ int walk_next(const Dims& dm, const Workspace& ws, Walk& k, uint16_t* list, int MT,
                         int lane) {
  int n = 0;
  while (k.left > 0) {
    if (k.w >= k.words) {  // unit finished: next pass, or the next group with rows
      k.w = 0;
      k.m = ~0u;
      ++k.serial;
      if (++k.p >= k.passes) {
        k.p = 0;
        bool ok;
        do {
          ++k.i;
          ok = walk_load_group(dm, ws, k, MT);
        } while (ok && __ldcg(ws.union_cnt + k.g) == 0);
        if (!ok) {  // the union counts and the bitmaps disagree
          if (lane == 0) report_error(ws.status, kErrDeviceInvalid);
          k.left = 0;
          break;
        }
      }
      continue;
    }
    const int word = k.w + lane;
    uint32_t bits = word < k.words ? __ldcg(ws.union_bits + (size_t)k.g * dm.fw + word) : 0u;
    if (lane == 0) bits &= k.m;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    const int excl = incl - c;
    const int cap = min(kListRows, k.left);
    const int take = min(max(cap - excl, 0), c);  // this lane's rows: its lowest `take` bits
    uint32_t bb = bits;
    int pos = excl;
    for (int t = 0; t < take; ++t) {
      list[pos++] = static_cast<uint16_t>(32 * word + __ffs(bb) - 1);
      bb &= bb - 1;
    }
    // the first lane that did not take all of its word holds the cursor
    const unsigned short_lanes = __ballot_sync(0xffffffffu, take < c);
    n = min(cap, __shfl_sync(0xffffffffu, incl, 31));
    if (short_lanes) {
      const int l = __ffs(short_lanes) - 1;
      k.m = __shfl_sync(0xffffffffu, bb, l);  // the rows of that word not taken yet
      k.w += l;
    } else {
      k.w += 32;
      k.m = ~0u;
    }
    k.left -= n;
    if (n > 0) break;
  }
  __syncwarp();  // list entries are read by every lane
  return n;
}

// The CTA's share of rows and where it starts. Every thread calls it.
__device__ void find_start(const Dims& dm, const Workspace& ws, int MT, Start* st,
                           long long* sm_warp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x / 32;
  // the first list entries are read while the list length is still in
  // flight (they are inside the list's capacity either way)
  const int g_spec = tid < dm.groups_max ? __ldcg(ws.gemv_list + tid) : 0;
  const int n_gv = min(__ldcg(ws.meta + kMetaGemvCount), kListMax);
  // rows of each GEMV group (all passes); one sweep when the groups fit the
  // CTA, else a first sweep for the total
  const bool one = n_gv <= (int)blockDim.x;
  long long lo = 0;
  if (tid == 0) {
    st->i = -1;
    st->rows = 0;
  }
  for (int sweep = one ? 1 : 0; sweep < 2; ++sweep) {
    long long carry = 0;
    for (int base = 0; base < n_gv; base += blockDim.x) {
      const int i = base + tid;
      long long v = 0;
      int g = 0, cnt = 0, words = 0;
      if (i < n_gv) {
        g = base == 0 ? g_spec : __ldcg(ws.gemv_list + i);
        cnt = __ldcg(ws.union_cnt + g);
        const Group gr = ws.groups[g];
        v = (long long)((gr.m + MT - 1) / MT) * cnt;
        words = (gr.expert >= dm.E ? dm.Fs : dm.F) / 32;
      }
      long long incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (lane == 31) sm_warp[warp] = incl;
      __syncthreads();
      long long before = 0, chunk = 0;
      for (int w = 0; w < nw; ++w) {
        const long long x = sm_warp[w];
        if (w < warp) before += x;
        chunk += x;
      }
      const long long excl = carry + before + incl - v;
      if (sweep == 1) {
        if (one) {  // the total is known now
          lo = chunk * blockIdx.x / gridDim.x;
          if (tid == 0) st->rows = (int)(chunk * (blockIdx.x + 1) / gridDim.x - lo);
        }
        if (v > 0 && excl <= lo && lo < excl + v) {
          const long long off = lo - excl;
          st->i = i;
          st->p = (int)(off / cnt);
          st->g = g;
          st->row = (int)(off % cnt);
          st->w = words;  // the group's word count, until warp 0 positions the cursor
        }
      }
      carry += chunk;
      __syncthreads();
    }
    if (sweep == 0) {
      lo = carry * blockIdx.x / gridDim.x;
      if (tid == 0) st->rows = (int)(carry * (blockIdx.x + 1) / gridDim.x - lo);
    }
  }
  __syncthreads();
  if (st->rows <= 0 || st->i < 0) return;  // uniform
  // warp 0: the bitmap word holding row st->row of group st->g
  if (warp == 0) {
    const int g = st->g, words = st->w;
    int skip = st->row;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const uint32_t bits =
          w0 + lane < words ? __ldcg(ws.union_bits + (size_t)g * dm.fw + w0 + lane) : 0u;
      const int c = __popc(bits);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      const int excl = incl - c;
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      __syncwarp();  // every lane has read st->w before the owner lane rewrites it
      if (excl <= skip && skip < incl) {  // this lane's word holds the first row
        uint32_t m = bits;
        for (int t = 0; t < skip - excl; ++t) m &= m - 1;  // drop the rows before it
        st->w = w0 + lane;
        st->m = m;
      }
      if (skip < total) break;
      skip -= total;
    }
  }
  __syncthreads();
}

template <typename TW>
struct Rows;

// bf16: tensor-core multiply of the landed rows.
template <>
struct Rows<__nv_bfloat16> {
  static constexpr int MT = kGemvTokens;  // tokens per pass
  static constexpr int kTiles = 16;       // 16-column tiles of the warp's 256 columns
  float acc[kTiles][4];

  __device__ void zero() {
#pragma unroll
    for (int i = 0; i < kTiles; ++i)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[i][v] = 0.f;
  }
  // D[16 columns][8 tokens] += W^T[16 columns][8 rows] * H[8 rows][8 tokens];
  // tokens >= mt and rows >= cnt enter as zero h.
  __device__ void consume(uint32_t rows_s, const uint8_t*, int stride, const uint8_t* hs, int cnt,
                          int mt, int lane) {
    const int g = lane >> 2, c2 = 2 * (lane & 3);
    uint32_t hb2 = 0u;  // H[rows c2, c2 + 1][token g]
    if (g < mt) {
      const uint32_t lo = c2 < cnt ? reinterpret_cast<const uint16_t*>(hs + c2 * kHBytes)[g] : 0u;
      const uint32_t hi =
          c2 + 1 < cnt ? reinterpret_cast<const uint16_t*>(hs + (c2 + 1) * kHBytes)[g] : 0u;
      hb2 = lo | (hi << 16);
    }
    const uint32_t row_s = rows_s + (lane & 7) * stride + (lane >> 3) * 16;
#pragma unroll
    for (int p = 0; p < kTiles / 2; ++p) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(row_s + p * 64, a0, a1, a2, a3);
      mma_16x8x8(acc[2 * p], a0, a1, hb2);
      mma_16x8x8(acc[2 * p + 1], a2, a3, hb2);
    }
  }
  // acc[i] = D[column 16i + g (+8)][tokens c2, c2 + 1]; lanes g and g ^ 1
  // swap halves so that each holds two adjacent columns of one token.
  // acc[i] = D[column 16i + g (+8)][tokens c2, c2 + 1] goes through the
  // warp's staging rows ys[token][kYStride] (row stride 260 floats: the four
  // token rows a store touches fall in different banks), then leaves as
  // 16-byte vector adds.
  __device__ void flush(float* y, int d, int mt, float* ys, int lane) {
    const int g = lane >> 2, c2 = 2 * (lane & 3);
#pragma unroll
    for (int i = 0; i < kTiles; ++i) {
      if (c2 < mt) {
        ys[c2 * kYStride + 16 * i + g] = acc[i][0];
        ys[c2 * kYStride + 16 * i + g + 8] = acc[i][2];
      }
      if (c2 + 1 < mt) {
        ys[(c2 + 1) * kYStride + 16 * i + g] = acc[i][1];
        ys[(c2 + 1) * kYStride + 16 * i + g + 8] = acc[i][3];
      }
    }
    __syncwarp();
    for (int t = 0; t < mt; ++t) {
#pragma unroll
      for (int h = 0; h < kTiles / 8; ++h) {
        const int col = 128 * h + 4 * lane;
        const float4 v = *reinterpret_cast<const float4*>(ys + t * kYStride + col);
        red_add_v4(y + (size_t)t * d + col, v.x, v.y, v.z, v.w);
      }
    }
    __syncwarp();
  }
};

// fp32: packed fp32x2 FMAs, 4 columns per lane, up to 8 tokens.
template <>
struct Rows<float> {
  static constexpr int MT = 8;
  uint64_t acc[MT][2];

  __device__ void zero() {
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = 0ull;
  }
  __device__ void consume(uint32_t, const uint8_t* rows, int stride, const uint8_t* hs, int cnt,
                          int mt, int lane) {
    for (int r = 0; r < cnt; ++r) {
      const float* hr = reinterpret_cast<const float*>(hs + r * kHBytes);
      const uint4 u = *reinterpret_cast<const uint4*>(rows + r * stride + lane * 16);
      const uint64_t w0 = pack2(__uint_as_float(u.x), __uint_as_float(u.y));
      const uint64_t w1 = pack2(__uint_as_float(u.z), __uint_as_float(u.w));
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t < mt) {
          const uint64_t h2 = pack2(hr[t], hr[t]);
          fma2(acc[t][0], h2, w0);
          fma2(acc[t][1], h2, w1);
        }
      }
    }
  }
  __device__ void flush(float* y, int d, int mt, float*, int lane) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t < mt) {
        const float2 a = unpack2(acc[t][0]), b = unpack2(acc[t][1]);
        red_add_v4(y + (size_t)t * d + lane * 4, a.x, a.y, b.x, b.y);
      }
    }
  }
};

template <typename TW>
__global__ void __launch_bounds__(kThreads, 1)
    down_gemv_kernel(Dims dm, Workspace ws, const TW* __restrict__ Wd,
                     const TW* __restrict__ Wds) {
  using R = Rows<TW>;
  constexpr int MT = R::MT;
  constexpr int ES = static_cast<int>(sizeof(TW));
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Start start;
  __shared__ long long sm_warp[kThreads / 32];
  __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ uint16_t list[kListRows];
  __shared__ int abort_flag;

  grid_dep_wait();
  find_start(dm, ws, MT, &start, sm_warp);
  if (start.rows <= 0 || start.i < 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = dm.d;
  const int row_bytes = d * ES;
  const Geometry geo = geometry(row_bytes);
  const int NS = geo.n_stages;
  const int n_blocks = (row_bytes + kBlockBytes - 1) / kBlockBytes;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NS; ++b) {
      mbar_init(full + b, 1 + kBatch);  // expect_tx arrival + one per h-copying lane
      mbar_init(empty + b, kConsumers);
    }
    abort_flag = 0;
    fence_barrier_init();
    atomicAdd(ws.counters + kCntDownRows, static_cast<unsigned long long>(start.rows));
  }
  __syncthreads();
  const uint32_t smem_s = smem_u32(smem);

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    // run-major: each run of rows (one unit) is streamed once per column
    // block, so the bitmaps are walked once
    const size_t ld = static_cast<size_t>(dm.slots_total);
    const char* ht = static_cast<const char*>(ws.ht);
    Walk k;
    k.i = start.i;
    k.p = start.p;
    k.w = start.w;
    k.m = start.m;
    k.left = start.rows;
    k.n_gv = min(__ldcg(ws.meta + kMetaGemvCount), kListMax);
    k.serial = 0;
    walk_load_group(dm, ws, k, MT);
    int s = 0;  // stages filled
    bool ok = true;
    for (bool last = false; ok && !last;) {
      const int n_list = walk_next(dm, ws, k, list, MT, lane);
      last = n_list == 0;
      const int slot = k.slot0 + k.p * MT;
      const int mt = min(MT, k.m_tok - k.p * MT);
      const TW* wexp = k.expert >= dm.E ? Wds + (size_t)(k.expert - dm.E) * dm.Fs * d
                                        : Wd + (size_t)k.expert * dm.F * d;
      for (int cb = 0; cb < (last ? 1 : n_blocks) && ok; ++cb) {
        const int cbytes = min(kBlockBytes, row_bytes - cb * kBlockBytes);
        for (int pos = 0; pos < n_list || (last && pos == 0); pos += kBatch) {
          const int b = s % NS;
          if (s >= NS && !warp_wait(empty + b, ((s / NS) + 1) & 1, &abort_flag, ws.status, kTight)) {
            ok = false;
            break;
          }
          uint8_t* stg = smem + b * geo.stage;
          const uint32_t stg_s = smem_s + b * geo.stage;
          const int cnt = last ? 0 : min(kBatch, n_list - pos);  // 0: the end marker
          if (!last && cnt < kBatch) {
            // rows past the run enter the mma with zero h: give them finite
            // values (never-written shared memory may hold any bits)
            for (int r = cnt; r < kBatch; ++r)
              for (int o = lane * 16; o < geo.block; o += 32 * 16)
                *reinterpret_cast<uint4*>(stg + r * geo.stride + o) = make_uint4(0u, 0u, 0u, 0u);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          }
          // stage metadata, then one arrival with the rows' transaction
          // bytes; lanes 0..7 copy the h values of their rows with cp.async
          // and arrive when those land (the consumers mask tokens past the
          // pass and rows past the run)
          if (lane == 0) {
            *reinterpret_cast<int4*>(stg + kBatch * geo.stride + kBatch * kHBytes) =
                make_int4(last ? -1 : k.serial * n_blocks + cb, cnt, slot, mt | (cb << 8));
            mbar_arrive_expect_tx(full + b, static_cast<uint32_t>(cnt * cbytes));
          }
          __syncwarp();
          if (lane < kBatch) {
            if (lane < cnt) {
              const int j = list[pos + lane];
              const uint32_t hdst = stg_s + kBatch * geo.stride + lane * kHBytes;
              const char* hsrc = ht + ((size_t)j * ld + slot) * ES;
              if constexpr (ES == 2) {
                cp_async8(hdst, hsrc);
              } else {
                cp_async16(hdst, hsrc);
                cp_async16(hdst + 16, hsrc + 16);
              }
              bulk_load(stg_s + lane * geo.stride,
                        wexp + (size_t)j * d + cb * (kBlockBytes / ES), cbytes,
                        smem_u32(full + b));
            }
            cp_async_arrive(smem_u32(full + b));
          }
          ++s;
        }
      }
    }
    // do not leave with copies in flight: wait (bounded) for the last stages
    if (!ok) {
      for (int q = max(0, s - NS); q < s; ++q)
        warp_wait(full + q % NS, (q / NS) & 1, &abort_flag, ws.status);
    }
  } else {
    // ------------------------------------------------------------ consumers
    R rows;
    float* ystage = reinterpret_cast<float*>(smem + NS * geo.stage) + warp * (kYBytes / 4);
    rows.zero();
    int cur_tag = -1, cur_slot = 0, cur_mt = 0, cur_col0 = 0;
    for (int s = 0;; ++s) {
      const int b = s % NS;
      if (!warp_wait(full + b, (s / NS) & 1, &abort_flag, ws.status, kTight)) break;
      const uint8_t* stg = smem + b * geo.stage;
      const int4 meta = *reinterpret_cast<const int4*>(stg + kBatch * geo.stride + kBatch * kHBytes);
      const int cb = meta.w >> 8, mt = meta.w & 255;
      const int cbytes = min(kBlockBytes, row_bytes - cb * kBlockBytes);
      // this warp's slice of the block; with narrow blocks several warps
      // share a slice and take alternate stages
      const int n_slices = cbytes / kSliceBytes;
      const int n_phase = n_slices >= kConsumers ? 1 : kConsumers / n_slices;
      const int slice = warp % n_slices, phase = warp / n_slices;
      const bool mine = phase < n_phase && (s % n_phase) == phase;
      if (meta.x != cur_tag && (mine || meta.x < 0)) {
        if (cur_tag >= 0) {
          rows.flush(ws.y + (size_t)cur_slot * d + cur_col0, d, cur_mt, ystage, lane);
          rows.zero();
        }
        cur_tag = meta.x;
        cur_slot = meta.z;
        cur_mt = mt;
        cur_col0 = (cb * kBlockBytes + slice * kSliceBytes) / ES;
      }
      if (mine && meta.y > 0)
        rows.consume(smem_s + b * geo.stage + slice * kSliceBytes, stg + slice * kSliceBytes,
                     geo.stride, stg + kBatch * geo.stride, meta.y, mt, lane);
      __syncwarp();  // every lane has read the stage
      if (lane == 0) mbar_arrive(empty + b);
      if (meta.x < 0) break;
    }
  }
}

}  // namespace

size_t down_gemv_smem_bytes(int d, bool bf16) {
  const Geometry g = geometry(d * (bf16 ? 2 : 4));
  return static_cast<size_t>(g.n_stages) * g.stage + (bf16 ? kConsumers * kYBytes : 0);
}

cudaError_t launch_down_gemv(const Dims& dm, const Workspace& ws, const void* Wd,
                             const void* Wds, bool bf16, int n_sms, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(down_gemv_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBudget + kConsumers * kYBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(down_gemv_kernel<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemBudget + kConsumers * kYBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = n_sms;  // one CTA per SM
  const size_t smem = down_gemv_smem_bytes(dm.d, bf16);
  if (bf16)
    return launch_k(down_gemv_kernel<__nv_bfloat16>, grid, kThreads, smem, st, dm, ws,
                    static_cast<const __nv_bfloat16*>(Wd), static_cast<const __nv_bfloat16*>(Wds));
  return launch_k(down_gemv_kernel<float>, grid, kThreads, smem, st, dm, ws,
                  static_cast<const float*>(Wd), static_cast<const float*>(Wds));
}

}  // namespace moe
