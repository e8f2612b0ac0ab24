// Sparse up projection of the gate-score variant for expert token groups
// with few tokens (decode): only the W_up rows of the group's active-row
// union are read, u_j = x . W_up[e][j, :] is formed for the pass's tokens,
// and h_j = SiLU(g_j) u_j replaces the masked SiLU(g_j) that the gate kernel
// left in H^T (zero for a token whose neuron is inactive), ready for the
// sparse down projection.
//
// The pages' system scores neurons by the dense gate projection alone and
// then fetches only the active neurons' up and down weights [gist.science EN
// "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-
// Expert Model Execution", Technical Summary > Methodology > System
// Implementation in vLLM > "Gate Projection", "Fused Up-Down Projection"].
// Here the up and down halves are two row-streaming kernels over the same
// row sequence; each reads every active row of its matrix once.
//
// Work split and producer: as in the down projection (gemv_common.cuh), the
// GEMV units' union rows are split evenly over the CTAs and a producer warp
// brings each row's 4 KB column block in with one bulk copy per row. The
// stage carries the rows' neuron indices instead of h values.
//
// Consumers: the 8 warps take 512-byte column slices of the block. For a
// stage of 8 rows each warp forms the partial dots of its slice on the tensor
// cores (mma.sync m16n8k16: 8 rows padded to 16 x 16 columns x up to 8
// tokens; the x values of the pass stay in registers while the unit and
// block are unchanged); the 8 partials are summed in warp order through
// shared memory and added, block after block, into the run's dot
// accumulators; after the run's last block the warps write
// h = SiLU(g) * u for the run's rows. All sums are in a fixed order.
#include "gemv_common.cuh"

namespace moe {

namespace {

constexpr int kMetaBytes = 48;  // per stage after the rows: 2 x int4 + 8 row indices
constexpr int kTok = 8;         // token columns of the mma (passes hold up to 8)

// d += A (16 x 16, bf16) * B (16 x 8, bf16), fp32 accumulation; rows 8..15
// of A are zero here.
__device__ __forceinline__ void mma_16x8x16(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                            uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// Two 8x8 bf16 matrices from shared memory (lanes 0..15 supply the row addresses).
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

template <typename TW>
struct UpDots;

// bf16: 16 K-steps of 16 columns over the warp's 256 columns.
template <>
struct UpDots<__nv_bfloat16> {
  static constexpr int MT = kGemvTokens;
  uint32_t xb[16][2];  // B fragments: x[token g][columns of K-step ks]

  // x values of the pass's tokens for this warp's columns [col0, col0 + 256)
  __device__ void load_x(const __nv_bfloat16* xrows, int d, int mt, int col0, int lane) {
    const int g = lane >> 2, c2 = 2 * (lane & 3);
    const __nv_bfloat16* xr = xrows + (size_t)g * d + col0 + c2;
#pragma unroll
    for (int ks = 0; ks < 16; ++ks) {
      xb[ks][0] = g < mt ? __ldcg(reinterpret_cast<const unsigned int*>(xr + 16 * ks)) : 0u;
      xb[ks][1] = g < mt ? __ldcg(reinterpret_cast<const unsigned int*>(xr + 16 * ks + 8)) : 0u;
    }
  }
  // partial dots of the stage's 8 rows over this warp's slice: p[0..1] =
  // (row g, tokens c2, c2 + 1)
  __device__ void dots(uint32_t rows_s, const uint8_t*, int stride, float (&p)[2], int lane) {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t a_addr = rows_s + (lane & 7) * stride + ((lane >> 3) & 1) * 16;
#pragma unroll
    for (int ks = 0; ks < 16; ++ks) {
      uint32_t a0, a2;
      ldsm_x2(a_addr + 32 * ks, a0, a2);
      mma_16x8x16(d, a0, a2, xb[ks][0], xb[ks][1]);
    }
    p[0] = d[0];
    p[1] = d[1];
  }
  // where this lane's two partials go: (row, token) pairs
  __device__ static void owner(int lane, int i, int& row, int& tok) {
    row = lane >> 2;
    tok = 2 * (lane & 3) + i;
  }
};

// fp32: 4 columns per lane, warp reduction per (row, token).
template <>
struct UpDots<float> {
  static constexpr int MT = 8;
  float xv[MT][4];

  __device__ void load_x(const float* xrows, int d, int mt, int col0, int lane) {
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        xv[t][i] = t < mt ? __ldcg(xrows + (size_t)t * d + col0 + 4 * lane + i) : 0.f;
  }
  __device__ void dots(uint32_t, const uint8_t* rows, int stride, float (&p)[2], int lane) {
    // 64 (row, token) sums; lane l ends with those of (row l / 8, tokens ..)
    p[0] = p[1] = 0.f;
#pragma unroll 1
    for (int r = 0; r < kBatch; ++r) {
      const float4 w = *reinterpret_cast<const float4*>(rows + r * stride + lane * 16);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        float v = w.x * xv[t][0] + w.y * xv[t][1] + w.z * xv[t][2] + w.w * xv[t][3];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        // (row r, token t) -> lane 4 r + t / 2, slot t % 2
        if (lane == 4 * r + t / 2) p[t & 1] = v;
      }
    }
  }
  __device__ static void owner(int lane, int i, int& row, int& tok) {
    row = lane >> 2;
    tok = 2 * (lane & 3) + i;
  }
};

template <typename TW>
__global__ void __launch_bounds__(kThreads, 1)
    up_gemv_kernel(Dims dm, Workspace ws, const TW* __restrict__ Wu, const TW* __restrict__ Wus,
                   const TW* __restrict__ x) {
  using D = UpDots<TW>;
  constexpr int MT = D::MT;
  constexpr int ES = static_cast<int>(sizeof(TW));
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Start start;
  __shared__ long long sm_warp[kThreads / 32];
  __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ uint16_t list[kListRows];
  __shared__ uint16_t rowj[kListRows];          // the current run's neuron indices
  __shared__ float uacc[kListRows][kTok];       // the current run's dot products
  __shared__ float red[2][kConsumers][kBatch][kTok];  // one stage's partials per warp
  __shared__ int abort_flag;

  grid_dep_wait();
  find_start(dm, ws, MT, &start, sm_warp);
  if (start.rows <= 0 || start.i < 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = dm.d;
  const int row_bytes = d * ES;
  const Geometry geo = geometry(row_bytes, kMetaBytes);
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
  }
  __syncthreads();
  const uint32_t smem_s = smem_u32(smem);

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    Walk k;
    k.i = start.i;
    k.p = start.p;
    k.w = start.w;
    k.m = start.m;
    k.left = start.rows;
    k.n_gv = min(__ldcg(ws.meta + kMetaGemvCount), kListMax);
    k.serial = 0;
    walk_load_group(dm, ws, k, MT);
    int s = 0;
    bool ok = true;
    for (bool last_run = false; ok && !last_run;) {
      const int n_list = walk_next(dm, ws, k, list, MT, lane);
      last_run = n_list == 0;
      const int slot = k.slot0 + k.p * MT;
      const int mt = min(MT, k.m_tok - k.p * MT);
      const int shared = k.expert >= dm.E;
      const TW* wexp = shared ? Wus + (size_t)(k.expert - dm.E) * dm.Fs * d
                              : Wu + (size_t)k.expert * dm.F * d;
      for (int cb = 0; cb < (last_run ? 1 : n_blocks) && ok; ++cb) {
        const int cbytes = min(kBlockBytes, row_bytes - cb * kBlockBytes);
        for (int pos = 0; pos < n_list || (last_run && pos == 0); pos += kBatch) {
          const int b = s % NS;
          if (s >= NS && !warp_wait(empty + b, ((s / NS) + 1) & 1, &abort_flag, ws.status, kTight)) {
            ok = false;
            break;
          }
          uint8_t* stg = smem + b * geo.stage;
          const uint32_t stg_s = smem_s + b * geo.stage;
          const int cnt = last_run ? 0 : min(kBatch, n_list - pos);  // 0: the end marker
          const int last = !last_run && cb == n_blocks - 1 && pos + cnt >= n_list;
          if (lane == 0) {
            int4* meta = reinterpret_cast<int4*>(stg + kBatch * geo.stride);
            meta[0] = make_int4(last_run ? -1 : k.serial * n_blocks + cb, cnt, slot,
                                mt | (cb << 8) | (last << 16));
            meta[1] = make_int4(pos, k.xrow0 + k.p * MT, shared, n_list);
            uint16_t* rj = reinterpret_cast<uint16_t*>(meta + 2);
            for (int r = 0; r < kBatch; ++r) rj[r] = r < cnt ? list[pos + r] : 0;
            mbar_arrive_expect_tx(full + b, static_cast<uint32_t>(cnt * cbytes));
          }
          __syncwarp();
          if (lane < cnt)
            bulk_load(stg_s + lane * geo.stride,
                      wexp + (size_t)list[pos + lane] * d + cb * (kBlockBytes / ES), cbytes,
                      smem_u32(full + b));
          ++s;
        }
      }
    }
    if (!ok) {  // do not leave with copies in flight
      for (int q = max(0, s - NS); q < s; ++q)
        warp_wait(full + q % NS, (q / NS) & 1, &abort_flag, ws.status);
    }
  } else {
    // ------------------------------------------------------------ consumers
    D dots;
    const size_t ld = static_cast<size_t>(dm.slots_total);
    TW* ht = static_cast<TW*>(ws.ht);
    int cur_tag = -2;
    bool ok = true;
    for (int s = 0;; ++s) {
      const int b = s % NS;
      // a failed wait is shared through the abort flag; the warps still meet
      // at every named barrier below, so none waits for a warp that left
      if (ok && !warp_wait(full + b, (s / NS) & 1, &abort_flag, ws.status, kTight)) ok = false;
      int4 m0 = make_int4(-1, 0, 0, 0), m1 = make_int4(0, 0, 0, 0);
      const uint8_t* stg = smem + b * geo.stage;
      if (ok) {
        const int4* meta = reinterpret_cast<const int4*>(stg + kBatch * geo.stride);
        m0 = meta[0];
        m1 = meta[1];
      }
      const int tag = m0.x, cnt = m0.y, slot = m0.z;
      const int mt = m0.w & 255, cb = (m0.w >> 8) & 255, last = (m0.w >> 16) & 1;
      const int pos = m1.x, xrow = m1.y, shared = m1.z, n_list = m1.w;
      float p[2] = {0.f, 0.f};
      if (tag >= 0) {
        const int cbytes = min(kBlockBytes, row_bytes - cb * kBlockBytes);
        const int n_slices = cbytes / kSliceBytes;
        if (warp < n_slices) {
          const int col0 = (cb * kBlockBytes + warp * kSliceBytes) / ES;
          if (tag != cur_tag) {
            const TW* xs = (shared ? x : static_cast<const TW*>(ws.xperm)) + (size_t)xrow * d;
            dots.load_x(xs, d, mt, col0, lane);
            cur_tag = tag;
          }
          dots.dots(smem_s + b * geo.stage + warp * kSliceBytes, stg + warp * kSliceBytes,
                    geo.stride, p, lane);
        }
        if (cb == 0 && warp == 0 && lane < cnt)
          rowj[pos + lane] = reinterpret_cast<const uint16_t*>(stg + kBatch * geo.stride + 32)[lane];
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        int r, t;
        D::owner(lane, i, r, t);
        red[s & 1][warp][r][t] = p[i];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + b);
      // one decision for all consumer warps: stop at the end marker or once
      // any warp's wait has failed
      if (consumers_any(tag < 0 || !ok)) break;
      // the stage's dots, summed over the warps in warp order
      if (threadIdx.x < kBatch * kTok) {
        const int r = threadIdx.x / kTok, t = threadIdx.x % kTok;
        if (r < cnt && t < mt) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumers; ++w) v += red[s & 1][w][r][t];
          uacc[pos + r][t] = cb == 0 ? v : uacc[pos + r][t] + v;
        }
      }
      if (last) {
        consumers_sync();
        // h = SiLU(g) u for the run's rows; H^T holds the masked SiLU(g)
        for (int i = threadIdx.x; i < n_list * mt; i += kConsumers * 32) {
          const int r = i / mt, t = i % mt;
          TW* hp = ht + (size_t)rowj[r] * ld + slot + t;
          const float sg = to_f32(*hp);
          *hp = from_f32<TW>(sg * uacc[r][t]);
        }
        consumers_sync();
      }
    }
  }
}

}  // namespace

size_t up_gemv_smem_bytes(int d, bool bf16) {
  const Geometry g = geometry(d * (bf16 ? 2 : 4), kMetaBytes);
  return static_cast<size_t>(g.n_stages) * g.stage;
}

cudaError_t launch_up_gemv(const Dims& dm, const Workspace& ws, const void* Wu, const void* Wus,
                           const void* x, bool bf16, int n_sms, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(up_gemv_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(up_gemv_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemBudget);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const size_t smem = up_gemv_smem_bytes(dm.d, bf16);
  if (bf16)
    return launch_k(up_gemv_kernel<__nv_bfloat16>, n_sms, kThreads, smem, st, dm, ws,
                    static_cast<const __nv_bfloat16*>(Wu), static_cast<const __nv_bfloat16*>(Wus),
                    static_cast<const __nv_bfloat16*>(x));
  return launch_k(up_gemv_kernel<float>, n_sms, kThreads, smem, st, dm, ws,
                  static_cast<const float*>(Wu), static_cast<const float*>(Wus),
                  static_cast<const float*>(x));
}

}  // namespace moe
