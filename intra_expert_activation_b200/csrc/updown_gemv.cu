// Fused sparse up + down projection of the gate-score variant for expert
// token groups with few tokens (decode). For each active row j of a group's
// union (neurons with |SiLU(g_j)| > tau for some token of the pass) it reads
// W_up[e][j, :] and W_down[e][j, :] once:
//   u_j = x . W_up[e][j, :],  h_j = SiLU(g_j) u_j  (zero where inactive),
//   y  += h_j W_down[e][j, :].
// The pages' system scores the neurons with the dense gate projection alone
// and then fetches only the active neurons' up and down weights in one fused
// step [gist.science EN "Uncovering Intra-expert Activation Sparsity for
// Efficient Mixture-of-Expert Model Execution", Technical Summary >
// Methodology > System Implementation in vLLM > "Gate Projection", "Fused
// Up-Down Projection"]; the gate/up kernel left the masked SiLU(g) in H^T.
//
// Work split and producer: the GEMV units' union rows are split evenly over
// the CTAs and a producer warp walks them in runs of up to 256 rows of one
// unit (gemv_common.cuh). For each run it streams the rows' W_up blocks
// (4 KB column blocks, one bulk copy per row) and then the same rows' W_down
// blocks through one ring of stages.
//
// Consumers (8 warps, 512-byte column slices): on a W_up stage each warp forms
// the partial dots of its slice (mma.sync m16n8k16), the partials are summed
// in warp order through shared memory and added, block after block, into the
// run's dot array; after the run's last W_up block the array is turned into h
// in place. On a W_down stage each warp accumulates h x W_down for its slice
// (mma.sync m16n8k8, h rounded to bf16 as the separate kernels do) and adds
// the partial sums of a unit into Y[slot][columns] with vector fp32 atomics
// when the unit or the column block changes (partials from several SMs meet
// there in arrival order). The consumer warps take every stage in step, with
// one decision per stage about stopping, so that a failed wait anywhere
// stops all of them.
#include "gemv_consumers.cuh"

namespace moe {

namespace {

constexpr int kStageRowsMax = 16;  // rows per stage: 16 (bf16), 8 (fp32)
constexpr int kMetaBytes = 32 + 2 * kStageRowsMax;  // per stage after the rows: 2 x int4 + row indices
constexpr int kKindDown = 1 << 17;

template <typename TW>
__global__ void __launch_bounds__(kThreads, 1)
    updown_gemv_kernel(Dims dm, Workspace ws, const TW* __restrict__ Wu,
                       const TW* __restrict__ Wus, const TW* __restrict__ Wd,
                       const TW* __restrict__ Wds, const TW* __restrict__ x) {
  using U = UpDots<TW>;
  using R = Rows<TW>;
  constexpr int MT = U::MT;
  // rows per stage: the up dots' mma M (bf16: 16), 8 for fp32; the down
  // projection takes a stage's rows 8 at a time (its mma's K)
  constexpr int RB = U::kRows;
  static_assert(RB % kBatch == 0 && RB <= kStageRowsMax, "stage rows");
  static_assert(R::MT == MT, "tokens per pass");
  constexpr int ES = static_cast<int>(sizeof(TW));
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Start start;
  __shared__ long long sm_warp[kThreads / 32];
  __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ uint16_t list[kListRows];
  __shared__ uint16_t rowj[kListRows];              // the current run's neuron indices
  __shared__ float hrun[kListRows][kTokStride];      // the run's dots, then its h values
  __shared__ float red[2][kConsumers][RB][kTok];  // one stage's partial dots per warp
  __shared__ int abort_flag;

  grid_dep_wait();
  find_start(dm, ws, MT, &start, sm_warp);
  if (start.rows <= 0 || start.i < 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = dm.d;
  const int row_bytes = d * ES;
  const Geometry geo = geometry(row_bytes, kMetaBytes, kBlockBytes, RB);
  const int NS = geo.n_stages;
  const int n_blocks = (row_bytes + kBlockBytes - 1) / kBlockBytes;
  if (threadIdx.x == 0) {
    for (int b = 0; b < NS; ++b) {
      mbar_init(full + b, 1);
      mbar_init(empty + b, kConsumers);
    }
    abort_flag = 0;
    fence_barrier_init();
    atomicAdd(ws.counters + kCntUpRows, static_cast<unsigned long long>(start.rows));
    atomicAdd(ws.counters + kCntDownRows, static_cast<unsigned long long>(start.rows));
    atomicAdd(ws.counters + kCntGemvRows, static_cast<unsigned long long>(start.rows));
  }
  __syncthreads();
  const uint32_t smem_s = smem_u32(smem);

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    Walk k;
    walk_begin(dm, ws, start, k, MT);
    int s = 0;
    bool ok = true;
    for (bool last_run = false; ok && !last_run;) {
      const int n_list = walk_next(dm, ws, k, list, MT, lane);
      last_run = n_list == 0;
      const int slot = k.slot0 + k.p * MT;
      const int mt = min(MT, k.m_tok - k.p * MT);
      const int shared = k.expert >= dm.E;
      const size_t eoff = shared ? (size_t)(k.expert - dm.E) * dm.Fs * d
                                 : (size_t)k.expert * dm.F * d;
      for (int phase = 0; phase < (last_run ? 1 : 2) && ok; ++phase) {  // W_up, then W_down
        const TW* wexp = (phase ? (shared ? Wds : Wd) : (shared ? Wus : Wu)) + eoff;
        for (int cb = 0; cb < (last_run ? 1 : n_blocks) && ok; ++cb) {
          const int cbytes = min(kBlockBytes, row_bytes - cb * kBlockBytes);
          for (int pos = 0; pos < n_list || (last_run && pos == 0); pos += RB) {
            const int b = s % NS;
            if (s >= NS &&
                !warp_wait(empty + b, ((s / NS) + 1) & 1, &abort_flag, ws.status, kTight)) {
              ok = false;
              break;
            }
            uint8_t* stg = smem + b * geo.stage;
            const uint32_t stg_s = smem_s + b * geo.stage;
            const int cnt = last_run ? 0 : min(RB, n_list - pos);  // 0: the end marker
            const int last_up = phase == 0 && cb == n_blocks - 1 && pos + cnt >= n_list;
            if (phase == 1 && cnt < RB) {
              // W_down rows past the run are the mma's K with zero h: give them
              // finite values (never-written shared memory may hold any bits)
              for (int r = cnt; r < RB; ++r)
                for (int o = lane * 16; o < geo.block; o += 32 * 16)
                  *reinterpret_cast<uint4*>(stg + r * geo.stride + o) = make_uint4(0u, 0u, 0u, 0u);
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
            if (lane == 0) {
              int4* meta = reinterpret_cast<int4*>(stg + RB * geo.stride);
              meta[0] = make_int4(last_run ? -1 : k.serial * n_blocks + cb, cnt, slot,
                                  mt | (cb << 8) | (last_up << 16) | (phase ? kKindDown : 0));
              meta[1] = make_int4(pos, k.xrow0 + k.p * MT, shared, n_list);
              uint16_t* rj = reinterpret_cast<uint16_t*>(meta + 2);
              for (int r = 0; r < RB; ++r) {
                const int j = r < cnt ? list[pos + r] : 0;
                rj[r] = moe_in_bounds(ws.status, j < 32 * k.words) ? j : 0;  // checked build: clamp
              }
              mbar_arrive_expect_tx(full + b, static_cast<uint32_t>(cnt * cbytes));
            }
            __syncwarp();
            if (lane < cnt) {
              int j = list[pos + lane];
              if (!moe_in_bounds(ws.status, j < 32 * k.words)) j = 0;  // checked build: clamp
              bulk_load(stg_s + lane * geo.stride, wexp + (size_t)j * d + cb * (kBlockBytes / ES),
                        cbytes, smem_u32(full + b));
            }
            ++s;
          }
        }
      }
    }
    if (!ok) {  // do not leave with copies in flight
      for (int q = max(0, s - NS); q < s; ++q)
        warp_wait(full + q % NS, (q / NS) & 1, &abort_flag, ws.status);
    }
  } else {
    // ------------------------------------------------------------ consumers
    U up;
    R down;
    down.zero();
    const size_t ld = static_cast<size_t>(dm.slots_total);
    const TW* ht = static_cast<const TW*>(ws.ht);
    int up_tag = -2;  // unit and block whose x values the warp holds
    int dn_tag = -1, dn_slot = 0, dn_mt = 0, dn_col0 = 0;  // unit and block being accumulated
    bool ok = true;
    for (int s = 0;; ++s) {
      const int b = s % NS;
      if (ok && !warp_wait(full + b, (s / NS) & 1, &abort_flag, ws.status, kTight)) ok = false;
      int4 m0 = make_int4(-1, 0, 0, 0), m1 = make_int4(0, 0, 0, 0);
      const uint8_t* stg = smem + b * geo.stage;
      if (ok) {
        const int4* meta = reinterpret_cast<const int4*>(stg + RB * geo.stride);
        m0 = meta[0];
        m1 = meta[1];
      }
      const int tag = m0.x, cnt = m0.y, slot = m0.z;
      const int mt = m0.w & 255, cb = (m0.w >> 8) & 255, last_up = (m0.w >> 16) & 1;
      const bool is_down = (m0.w & kKindDown) != 0;
      const int pos = m1.x, xrow = m1.y, shared = m1.z, n_list = m1.w;
      const int cbytes = min(kBlockBytes, row_bytes - cb * kBlockBytes);
      const int n_slices = cbytes / kSliceBytes;
      const bool active = warp < n_slices;
      const int col0 = (cb * kBlockBytes + warp * kSliceBytes) / ES;
      float p[U::kParts];
#pragma unroll
      for (int i = 0; i < U::kParts; ++i) p[i] = 0.f;
      if (tag >= 0 && !is_down) {
        if (active) {
          if (tag != up_tag) {
            const TW* xs = (shared ? x : static_cast<const TW*>(ws.xperm)) + (size_t)xrow * d;
            up.load_x(xs, d, mt, col0, lane);
            up_tag = tag;
          }
          up.dots(smem_s + b * geo.stage + warp * kSliceBytes, stg + warp * kSliceBytes,
                  geo.stride, p, lane);
        }
        if (cb == 0 && warp == 0 && lane < cnt)
          rowj[pos + lane] = reinterpret_cast<const uint16_t*>(stg + RB * geo.stride + 32)[lane];
#pragma unroll
        for (int i = 0; i < U::kParts; ++i) {
          int r, t;
          U::owner(lane, i, r, t);
          red[s & 1][warp][r][t] = p[i];
        }
      }
      if (dn_tag >= 0 && (tag < 0 || (is_down && active && tag != dn_tag))) {
        down.flush(ws.y + (size_t)dn_slot * d + dn_col0, d, dn_mt, lane);
        down.zero();
        dn_tag = -1;
      }
      if (tag >= 0 && is_down && active) {
        if (tag != dn_tag) {
          dn_tag = tag;
          dn_slot = slot;
          dn_mt = mt;
          dn_col0 = col0;
        }
#pragma unroll
        for (int h = 0; h < RB / kBatch; ++h)  // the mma's K is 8 rows
          if (cnt > h * kBatch)
            down.consume_hf(smem_s + b * geo.stage + h * kBatch * geo.stride + warp * kSliceBytes,
                            stg + h * kBatch * geo.stride + warp * kSliceBytes, geo.stride,
                            &hrun[pos + h * kBatch][0], cnt - h * kBatch, mt, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + b);
      // one decision for all consumer warps: stop at the end marker or once
      // any warp's wait has failed
      if (consumers_any(tag < 0 || !ok)) break;
      if (!is_down) {
        // the stage's dots, summed over the warps in warp order
        if (threadIdx.x < RB * kTok) {
          const int r = threadIdx.x / kTok, t = threadIdx.x % kTok;
          if (r < cnt && t < mt) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumers; ++w) v += red[s & 1][w][r][t];
            hrun[pos + r][t] = cb == 0 ? v : hrun[pos + r][t] + v;
          }
        }
        if (last_up) {
          consumers_sync();
          // h = SiLU(g) u for the run's rows; H^T holds the masked SiLU(g)
          for (int i = threadIdx.x; i < n_list * MT; i += kConsumers * 32) {
            const int r = i / MT, t = i % MT;
            hrun[r][t] = t < mt ? to_f32(ht[(size_t)rowj[r] * ld + slot + t]) * hrun[r][t] : 0.f;
          }
          consumers_sync();
        }
      }
    }
    __syncwarp();
  }
}

}  // namespace

size_t updown_gemv_smem_bytes(int d, bool bf16) {
  const Geometry g = geometry(d * (bf16 ? 2 : 4), kMetaBytes, kBlockBytes, bf16 ? 16 : 8);
  return static_cast<size_t>(g.n_stages) * g.stage;
}

cudaError_t launch_updown_gemv(const Dims& dm, const Workspace& ws, const void* Wu,
                               const void* Wus, const void* Wd, const void* Wds, const void* x,
                               bool bf16, int n_sms, cudaStream_t st) {
  // dynamic shared memory as this launch needs it (the kernel's static
  // arrays come on top, so the attribute is raised to what is used only)
  const size_t smem = updown_gemv_smem_bytes(dm.d, bf16);
  const cudaError_t e = bf16 ? smem_limit(updown_gemv_kernel<__nv_bfloat16>, (int)smem)
                             : smem_limit(updown_gemv_kernel<float>, (int)smem);
  if (e != cudaSuccess) return e;
  if (bf16)
    return launch_k(updown_gemv_kernel<__nv_bfloat16>, n_sms, kThreads, smem, st, dm, ws,
                    static_cast<const __nv_bfloat16*>(Wu), static_cast<const __nv_bfloat16*>(Wus),
                    static_cast<const __nv_bfloat16*>(Wd), static_cast<const __nv_bfloat16*>(Wds),
                    static_cast<const __nv_bfloat16*>(x));
  return launch_k(updown_gemv_kernel<float>, n_sms, kThreads, smem, st, dm, ws,
                  static_cast<const float*>(Wu), static_cast<const float*>(Wus),
                  static_cast<const float*>(Wd), static_cast<const float*>(Wds),
                  static_cast<const float*>(x));
}

}  // namespace moe
