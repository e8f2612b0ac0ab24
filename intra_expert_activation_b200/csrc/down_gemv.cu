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
//
// Direct combine (dm.direct_combine: every group of the forward is on this
// path and T is small): the flush adds w x the sums of a slot straight into
// its token's output accumulator row Y[token] (w: the slot's combine weight,
// 1 for shared experts), and the last CTA to finish (a ticket) writes out
// from those rows, so no combine kernel runs.
#include "gemv_consumers.cuh"

namespace moe {

namespace {

constexpr int kStageExtra = kBatch * kHBytes + 16;   // per stage after the rows: h | meta

// Column blocks of this kernel. Wide (bf16 rows of a multiple of 1 KB,
// d_model % 512 == 0): rows up to 8 KB (d_model <= 4096) come in one bulk
// copy per row and each consumer warp owns a 1 KB slice (32 sixteen-column
// tiles); whole-row copies stream faster than two 4 KB halves fetched apart.
// Otherwise (fp32, and bf16 rows of an odd number of 512-byte slices): 4 KB
// blocks and 512-byte slices.
template <bool WIDE>
struct Blocks {
  static constexpr int kBlock = WIDE ? 8192 : kBlockBytes;
  static constexpr int kSlice = WIDE ? 1024 : kSliceBytes;
};
__host__ __device__ inline bool wide_rows(int d, bool bf16) { return bf16 && d % 512 == 0; }

// Where a consumer lane's sums of the current unit go under direct combine.
template <typename TW>
struct Direct;
template <>
struct Direct<__nv_bfloat16> {  // one token per lane (Rows::flush_token)
  float* row;
  float w;
  bool on;
  __device__ void load(const Dims& dm, const Workspace& ws, int slot, int mt, int col0, int lane) {
    const int t = Rows<__nv_bfloat16>::flush_token(lane);
    on = t < mt;
    row = ws.y;
    w = 0.f;
    if (on) {
      int tok;
      slot_target(dm, ws, slot + t, tok, w);
      row = ws.y + (size_t)tok * dm.d + col0;
    }
  }
  template <class R>
  __device__ void flush(R& r, int, int lane) {
    r.flush_to(row, w, on, lane);
  }
};
template <>
struct Direct<float> {  // every token of the pass per lane
  static constexpr int MT = Rows<float>::MT;
  float* row[MT];
  float w[MT];
  __device__ void load(const Dims& dm, const Workspace& ws, int slot, int mt, int col0, int) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      row[t] = ws.y;
      w[t] = 0.f;
      if (t < mt) {
        int tok;
        slot_target(dm, ws, slot + t, tok, w[t]);
        row[t] = ws.y + (size_t)tok * dm.d + col0;
      }
    }
  }
  template <class R>
  __device__ void flush(R& r, int mt, int lane) {
    r.flush_rows(row, w, mt, lane);
  }
};

template <typename TW, bool WIDE>
__global__ void __launch_bounds__(kThreads, 1)
    down_gemv_kernel(Dims dm, Workspace ws, const TW* __restrict__ Wd,
                     const TW* __restrict__ Wds, void* out, int out_bf16) {
  using B = Blocks<WIDE>;
  using R = Rows<TW, B::kSlice / 32>;
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
  if (start.rows <= 0 || start.i < 0) {  // uniform
    if (dm.direct_combine) direct_finish(dm, ws, out, out_bf16);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = dm.d;
  const int row_bytes = d * ES;
  const Geometry geo = geometry(row_bytes, kStageExtra, B::kBlock);
  const int NS = geo.n_stages;
  const int n_blocks = (row_bytes + B::kBlock - 1) / B::kBlock;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NS; ++b) {
      mbar_init(full + b, 1 + kBatch);  // expect_tx arrival + one per h-copying lane
      mbar_init(empty + b, kConsumers);
    }
    abort_flag = 0;
    fence_barrier_init();
    atomicAdd(ws.counters + kCntDownRows, static_cast<unsigned long long>(start.rows));
    atomicAdd(ws.counters + kCntGemvRows, static_cast<unsigned long long>(start.rows));
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
    walk_begin(dm, ws, start, k, MT);
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
        const int cbytes = min(B::kBlock, row_bytes - cb * B::kBlock);
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
              int j = list[pos + lane];
              if (!moe_in_bounds(ws.status, j < 32 * k.words && slot + MT <= dm.slots_total))
                j = 0;  // checked build: a bad row or slot is recorded and clamped
              const uint32_t hdst = stg_s + kBatch * geo.stride + lane * kHBytes;
              const char* hsrc = ht + ((size_t)j * ld + slot) * ES;
              if constexpr (ES == 2) {
                cp_async16(hdst, hsrc);  // 8 bf16 h values (slots of a pass are 16-B aligned)
              } else {
                cp_async16(hdst, hsrc);
                cp_async16(hdst + 16, hsrc + 16);
              }
              bulk_load(stg_s + lane * geo.stride,
                        wexp + (size_t)j * d + cb * (B::kBlock / ES), cbytes,
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
    rows.zero();
    Direct<TW> dir;
    int cur_tag = -1, cur_slot = 0, cur_mt = 0, cur_col0 = 0;
    for (int s = 0;; ++s) {
      const int b = s % NS;
      if (!warp_wait(full + b, (s / NS) & 1, &abort_flag, ws.status, kTight)) break;
      const uint8_t* stg = smem + b * geo.stage;
      const int4 meta = *reinterpret_cast<const int4*>(stg + kBatch * geo.stride + kBatch * kHBytes);
      const int cb = meta.w >> 8, mt = meta.w & 255;
      const int cbytes = min(B::kBlock, row_bytes - cb * B::kBlock);
      // this warp's slice of the block; with narrow blocks several warps
      // share a slice and take alternate stages
      const int n_slices = cbytes / B::kSlice;
      const int n_phase = n_slices >= kConsumers ? 1 : kConsumers / n_slices;
      const int slice = warp % n_slices, phase = warp / n_slices;
      const bool mine = phase < n_phase && (s % n_phase) == phase;
      if (meta.x != cur_tag && (mine || meta.x < 0)) {
        if (cur_tag >= 0) {
          if (dm.direct_combine)
            dir.flush(rows, cur_mt, lane);
          else
            rows.flush(ws.y + (size_t)cur_slot * d + cur_col0, d, cur_mt, lane);
          rows.zero();
        }
        cur_tag = meta.x;
        cur_slot = meta.z;
        cur_mt = mt;
        cur_col0 = (cb * B::kBlock + slice * B::kSlice) / ES;
        // the new unit's output rows and weights, loaded long before its flush
        if (dm.direct_combine && cur_tag >= 0) dir.load(dm, ws, cur_slot, cur_mt, cur_col0, lane);
      }
      if (mine && meta.y > 0)
        rows.consume(smem_s + b * geo.stage + slice * B::kSlice, stg + slice * B::kSlice,
                     geo.stride, stg + kBatch * geo.stride, meta.y, mt, lane);
      __syncwarp();  // every lane has read the stage
      if (lane == 0) mbar_arrive(empty + b);
      if (meta.x < 0) break;
    }
  }
  if (dm.direct_combine) direct_finish(dm, ws, out, out_bf16);
}

}  // namespace

size_t down_gemv_smem_bytes(int d, bool bf16) {
  const int block = wide_rows(d, bf16) ? Blocks<true>::kBlock : Blocks<false>::kBlock;
  const Geometry g = geometry(d * (bf16 ? 2 : 4), kStageExtra, block);
  return static_cast<size_t>(g.n_stages) * g.stage;
}

namespace {
template <typename TW, bool WIDE>
cudaError_t launch_dg(const Dims& dm, const Workspace& ws, const void* Wd, const void* Wds,
                      int n_sms, void* out, bool out_bf16, cudaStream_t st) {
  const cudaError_t e = smem_limit(down_gemv_kernel<TW, WIDE>, kSmemBudget);
  if (e != cudaSuccess) return e;
  const int grid = n_sms;  // one CTA per SM
  const size_t smem = down_gemv_smem_bytes(dm.d, sizeof(TW) == 2);
  return launch_k(down_gemv_kernel<TW, WIDE>, grid, kThreads, smem, st, dm, ws,
                  static_cast<const TW*>(Wd), static_cast<const TW*>(Wds), out, out_bf16 ? 1 : 0);
}
}  // namespace

cudaError_t launch_down_gemv(const Dims& dm, const Workspace& ws, const void* Wd,
                             const void* Wds, bool bf16, int n_sms, void* out, bool out_bf16,
                             cudaStream_t st) {
  if (!bf16) return launch_dg<float, false>(dm, ws, Wd, Wds, n_sms, out, out_bf16, st);
  if (wide_rows(dm.d, true))
    return launch_dg<__nv_bfloat16, true>(dm, ws, Wd, Wds, n_sms, out, out_bf16, st);
  return launch_dg<__nv_bfloat16, false>(dm, ws, Wd, Wds, n_sms, out, out_bf16, st);
}

}  // namespace moe
