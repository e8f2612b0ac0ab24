// Pieces shared by the row-streaming kernels of the decode path (the sparse
// down projection, and the sparse up projection of the gate-score variant):
// the equal split of the GEMV units' union rows over the CTAs, the producer
// warp's walk over the union bitmaps, and the copy / tensor-core helpers.
//
// The row sequence: a unit is (GEMV group, pass of up to MT of its tokens);
// its rows are the group's union rows (count in union_cnt, left by the
// gate/up epilogue). The units' rows in (group, pass, neuron) order form one
// sequence of R rows; CTA c (one per SM) takes rows [R c / G, R (c+1) / G).
#pragma once

#include "common.cuh"

namespace moe {
namespace {

constexpr int kConsumers = 8;
constexpr int kThreads = (kConsumers + 1) * 32;  // + the producer warp
constexpr int kBatch = 8;            // rows per stage (the mma's K)
constexpr int kSliceBytes = 512;     // row bytes per consumer warp (4 KB column blocks)
constexpr int kBlockBytes = kConsumers * kSliceBytes;  // column block: 4 KB of a row
constexpr int kRowPad = 16;          // row stride = block bytes + 16
constexpr int kMaxStages = 6;
constexpr int kSmemBudget = 200 * 1024;  // ring of stages (6 stages of 4 KB blocks)
constexpr int kListRows = 256;       // producer's row list (uint16 neuron indices)
constexpr int kTight = 4096;         // barrier probes before sleeping: stages arrive every few us

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// Arrive on bar once this thread's earlier cp.async copies have landed (the
// barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Stage geometry for a row of row_bytes: the column block (<= block_max),
// the stage size (`rows` rows, kBatch by default, at the padded stride, then
// `extra` bytes of per-stage data) and the number of stages that fit the
// budget.
struct Geometry {
  int block, stride, stage, n_stages;
};
__host__ __device__ inline Geometry geometry(int row_bytes, int extra,
                                             int block_max = kBlockBytes, int rows = kBatch) {
  Geometry g;
  g.block = row_bytes < block_max ? row_bytes : block_max;
  g.stride = g.block + kRowPad;
  g.stage = rows * g.stride + extra;
  g.n_stages = kSmemBudget / g.stage;
  if (g.n_stages > kMaxStages) g.n_stages = kMaxStages;
  return g;
}

// Named barrier 2 over the consumer warps (kConsumers x 32 threads), plain
// and with an OR of a predicate (every consumer thread gets the same answer).
static_assert(kConsumers == 8, "named barriers below count 256 threads");
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 2, 256;" ::: "memory"); }
__device__ __forceinline__ bool consumers_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 2, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// Where a CTA's share of the row sequence starts.
struct Start {
  int i;        // GEMV list index of the first group
  int p;        // pass within it
  int w;        // bitmap word of the first row
  uint32_t m;   // mask of the rows of word w that are still to come
  int rows;     // rows of this CTA
  int g, row;   // the first group and the row within its pass
  Group gr;     // the first group's record
};

// The producer's walk over its CTA's rows: group list index, pass, next word
// and the mask for it, rows still to produce, and the unit being produced.
struct Walk {
  int i, p, w;
  uint32_t m;
  int left;
  int n_gv;  // GEMV groups
  int g, words, passes, slot0, m_tok, expert, xrow0;  // unit data of group i
  int serial;  // increments whenever the unit (group, pass) changes
};

// Unit data of group g (record gr).
__device__ __forceinline__ void walk_set_group(const Dims& dm, Walk& k, int g, const Group& gr,
                                               int MT) {
  k.g = g;
  k.expert = gr.expert;
  k.slot0 = gr.slot0;
  k.m_tok = gr.m;
  k.xrow0 = gr.xrow0;
  k.passes = (gr.m + MT - 1) / MT;
  k.words = (gr.expert >= dm.E ? dm.Fs : dm.F) / 32;
}

// The producer's walk from the CTA's start (no global loads).
__device__ __forceinline__ void walk_begin(const Dims& dm, const Workspace& ws, const Start& st,
                                           Walk& k, int MT) {
  k.i = st.i;
  k.p = st.p;
  k.w = st.w;
  k.m = st.m;
  k.left = st.rows;
  k.n_gv = min(__ldcg(ws.meta + kMetaGemvCount), kListMax);
  k.serial = 0;
  walk_set_group(dm, k, st.g, st.gr, MT);
}

// Loads group i's unit data; false past the end of the GEMV list.
__device__ __forceinline__ bool walk_load_group(const Dims& dm, const Workspace& ws, Walk& k,
                                                int MT) {
  if (k.i >= k.n_gv) return false;
  k.g = __ldcg(ws.gemv_list + k.i);
  const Group gr = ws.groups[k.g];
  k.expert = gr.expert;
  k.slot0 = gr.slot0;
  k.m_tok = gr.m;
  k.xrow0 = gr.xrow0;
  k.passes = (gr.m + MT - 1) / MT;
  k.words = (gr.expert >= dm.E ? dm.Fs : dm.F) / 32;
  return true;
}

// Rows per pass of group k.g on this kernel: its union count, or 0 for a
// candidate group that the tensor-core path takes.
__device__ __forceinline__ int walk_unit_rows(const Workspace& ws, const Walk& k) {
  const int cnt = __ldcg(ws.union_cnt + k.g);
  if (__ldcg(ws.group_path + k.g) == kPathCand && !cand_takes_gemv(cnt, k.passes, 32 * k.words))
    return 0;
  return cnt;
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
        } while (ok && walk_unit_rows(ws, k) == 0);
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
      Group gr{};
      if (i < n_gv) {
        g = base == 0 ? g_spec : __ldcg(ws.gemv_list + i);
        cnt = __ldcg(ws.union_cnt + g);
        const int path = __ldcg(ws.group_path + g);
        gr = ws.groups[g];
        const int passes = (gr.m + MT - 1) / MT;
        words = (gr.expert >= dm.E ? dm.Fs : dm.F) / 32;
        if (path == kPathCand) {  // decided now, from its union (the TC kernel agrees)
          const bool take = cand_takes_gemv(cnt, passes, 32 * words);
          if (!take) cnt = 0;
          if (take && sweep == 1 && blockIdx.x == 0)
            atomicAdd(ws.counters + kCntGemv, 1ull);
        }
        v = (long long)passes * cnt;
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
          st->gr = gr;
          st->row = (int)(off % cnt);
          st->w = words;  // the group's word count, until the cursor is placed
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
  // the bitmap word holding row st->row of group st->g: every thread loads
  // one word of a window of blockDim words (all loads in flight together),
  // a CTA-wide prefix sum of their row counts finds the word
  const int g = st->g, words = st->w;
  int skip = st->row;
  int* cnt_w = reinterpret_cast<int*>(sm_warp);
  for (int w0 = 0; w0 < words; w0 += blockDim.x) {
    const int word = w0 + tid;
    const uint32_t bits = word < words ? __ldcg(ws.union_bits + (size_t)g * dm.fw + word) : 0u;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) cnt_w[warp] = incl;
    __syncthreads();  // also: every thread has read st->w before its owner rewrites it
    int before = 0, total = 0;
    for (int w = 0; w < nw; ++w) {
      const int x = cnt_w[w];
      if (w < warp) before += x;
      total += x;
    }
    const int excl = before + incl - c;
    if (excl <= skip && skip < excl + c) {  // this thread's word holds the first row
      uint32_t m = bits;
      for (int t = 0; t < skip - excl; ++t) m &= m - 1;  // drop the rows before it
      st->w = word;
      st->m = m;
    }
    __syncthreads();  // cnt_w is rewritten by the next window
    if (skip < total) break;  // uniform
    skip -= total;
  }
  __syncthreads();
}

}  // namespace
}  // namespace moe
