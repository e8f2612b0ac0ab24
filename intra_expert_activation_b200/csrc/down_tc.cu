// Down projection on the 5th-generation tensor cores, reading all W_down rows
// of an expert token group or only those of its active-neuron union.
//
// The pages' kernel gathers the weights of the active neurons, packs them
// densely in shared memory and multiplies densely [gist.science EN
// "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
// Model Execution", Technical Summary > Methodology > System Implementation in
// vLLM > "Fused Up-Down Projection"]. Here the packing is done by four gather
// warps with 16-byte cp.async copies: each union row's 256 bytes of the unit's
// columns land at their packed K position in the 128-byte-swizzled layout the
// MMA reads, so the tensor core sees a dense K-block of union rows.
//
// Work unit: (group, 128-column slice of d_model); K = the group's rows.
//   D[128 columns][N tokens] = W_down[e][K rows, slice]^T . H^T[K rows, group slots]
// Both operands are MN-major in shared memory: a W_down row is 128
// contiguous output columns (M), an H^T row is 64 contiguous slots (N).
//   all-rows mode: K-block = 64 consecutive rows, loaded by TMA in 64-row
//     boxes; h of inactive neurons is an exact zero, so the sum is the same.
//   gathered mode (groups of <= 64 tokens: forced, or in AUTO when the union
//     is at most gather_density x d_ff): K-block = the next 64 union rows.
//     Warp 0 walks the group's union bitmap (copied to shared memory once per
//     unit) and writes each K-block's row numbers into the next of kIxSlots
//     row slots (a ring that runs ahead of the copies); warps 6-9 copy 16
//     rows each (A: 16 x 256 B, B: 16 x N slots x 2 B) into the ring stage,
//     every lane arriving on the stage's gather barrier when its copies land,
//     and the MMA thread fences the async proxy before reading. Positions
//     past the union are zero-filled (src-size 0) in both operands.
//     (TMA tile::gather4 with one-row boxes, tried first, streamed at about a
//     third of HBM bandwidth: a CTA's gather copies went out one after the
//     other; sixteen-byte copies from four warps per CTA, two CTAs per SM,
//     stream at 5.6-6.1 TB/s in a copy-only probe.)
// Warp roles: warp 0 TMA / union walk, warp 1 MMA + TMEM owner, warps 2-5
// drain TMEM into Y[slot][col] (fp32), coalesced across lanes, warps 6-9
// gather copies.
// With few units for the grid (decode batches with one to a few groups on
// this path), a unit's K-blocks are cut into parts (tc_ksplit): each part
// drains its sums into a workspace block, and the part that finishes last
// (an atomic ticket per unit) adds the parts in part order and stores Y.
// A candidate group that the row stream takes (cand_takes_gemv) is skipped.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kGatherWarp0 = 6;  // warps 6..9 copy the gathered rows
constexpr int kGatherWarps = 4;
constexpr int kThreads = 32 * (kGatherWarp0 + kGatherWarps);
constexpr int kGatherRows = kKBlock / kGatherWarps;  // rows of a K-block per gather warp
// Union-row slots between warp 0 and the gather warps: the walk runs up to
// this many gathered K-blocks ahead of the copies, off the ring's round trip.
constexpr int kIxSlots = 16;

// The four epilogue warps (warps 2..5) only: named barrier 1, plain and as
// an AND vote (every thread gets the same answer).
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}
// Units in flight between the TMA warp, which takes them from the queue, and
// the MMA and epilogue warps, which process them in the same order.
constexpr int kUQ = 4;
struct UnitQueue {
  int id[kUQ];                 // unit of each slot, -1: the queue is empty
  uint64_t full[kUQ];          // the TMA warp published the slot (1 arrival)
  uint64_t empty[kUQ];         // the MMA, epilogue and gather warps read it (9 arrivals)
};

constexpr uint32_t kAAtom = 64 * 128;  // one 64-row x 128-byte swizzled atom column
constexpr uint32_t kABytes = 2 * kAAtom;

struct DownUnit {
  Group gr;
  int g;
  int slice;
  int k0;         // first K-block of this unit's part
  int part;       // K part of the unit (0 .. ks-1)
  int ub;         // (list index, slice) of the unit: its ticket
  int gather;     // 1: gathered rows, 0: all rows
  int auto_gather;  // gathered by the union rule here (AUTO), counted by this kernel
  int F_e;        // rows of the expert
  int nk;         // K-blocks
  int cnt;        // union rows (gathered)
  int row_base;   // first row of this expert in the 2-D [experts*F][d] view
  int shared;
  int cand;       // candidate group, decided from its union
  int skip;       // candidate taken by the GEMV kernel: no work, no Y writes here
};

// Unit u = ((list index, part), slice): the slices of one part of a group
// are consecutive units, so the CTAs that run at the same time read whole
// W_down rows between them (as without parts), not narrow strips of
// different rows.
__device__ __forceinline__ DownUnit decode(const DownTcParams& p, int u, int n_slices, int ks) {
  DownUnit du;
  du.slice = u % n_slices;
  u /= n_slices;
  const int part = u % ks;
  const int li = u / ks;
  du.part = part;
  du.ub = li * n_slices + du.slice;
  du.g = __ldcg(p.ws.tc_list + li);
  du.gr = p.ws.groups[du.g];
  du.shared = du.gr.expert >= p.dm.E;
  const int F_e = du.shared ? p.dm.Fs : p.dm.F;
  const int e_local = du.shared ? du.gr.expert - p.dm.E : du.gr.expert;
  du.row_base = e_local * F_e;
  const int path = __ldcg(p.ws.group_path + du.g);
  du.F_e = F_e;
  du.cnt = __ldcg(p.ws.union_cnt + du.g);
  // AUTO: a group on all rows whose union is at most gather_density x d_ff
  // reads only the union rows
  du.auto_gather = path == kPathTcAll && p.dm.gather_density > 0.f &&
                   du.gr.m <= kGatherMaxTokens &&
                   static_cast<float>(du.cnt) <= p.dm.gather_density * static_cast<float>(F_e);
  du.gather = path == kPathTcGather || du.auto_gather;
  du.cand = path == kPathCand;
  du.skip = du.cand && cand_takes_gemv(du.cnt, (du.gr.m + kGemvTokens - 1) / kGemvTokens, F_e);
  const int nk = du.skip ? 0 : du.gather ? (du.cnt + kKBlock - 1) / kKBlock : F_e / kKBlock;
  du.k0 = nk * part / ks;
  du.nk = nk * (part + 1) / ks - du.k0;
  return du;
}

// TMA warp: take the next unit from the queue and publish it in slot
// n % kUQ, once the MMA and epilogue warps have read that slot's previous
// unit. Returns the unit, -1 when the queue is empty (also published), or -2
// when a wait gave up.
__device__ __forceinline__ int uq_take(UnitQueue& uq, int n, int* queue, int n_units,
                                       volatile int* abort, int* status, int lane) {
  const int q = n % kUQ;
  if (n >= kUQ && !warp_wait(&uq.empty[q], ((n / kUQ) - 1) & 1, abort, status)) return -2;
  int u = 0;
  if (lane == 0) {
    u = atomicAdd(queue, 1);
    if (u >= n_units) u = -1;
    uq.id[q] = u;
    mbar_arrive(&uq.full[q]);
  }
  return __shfl_sync(0xffffffffu, u, 0);
}

// MMA and epilogue warps: the n-th unit of this CTA (-1: none left, -2: a
// wait gave up); the slot is released as soon as it is read.
__device__ __forceinline__ int uq_next(UnitQueue& uq, int n, volatile int* abort, int* status,
                                       int lane) {
  const int q = n % kUQ;
  if (!warp_wait(&uq.full[q], (n / kUQ) & 1, abort, status)) return -2;
  const int u = uq.id[q];
  __syncwarp();
  if (lane == 0) mbar_arrive(&uq.empty[q]);
  return u;
}

// Warp 0, gathered units: the union walk. The group's union bitmap is in
// shared memory (bm, `words` words); (ww, wrem) is the walk position: word ww,
// of which the bits in wrem are still to be taken (lane-uniform).
struct UnionWalk {
  int ww;
  uint32_t wrem;
};

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

__device__ __forceinline__ uint32_t drop_low_bits(uint32_t b, int k) {
  for (int i = 0; i < k; ++i) b &= b - 1;
  return b;
}

// The walk position of union position pos (0 <= pos < the union's rows).
__device__ __forceinline__ UnionWalk walk_seek(const uint32_t* bm, int words, int pos, int lane) {
  UnionWalk w{words, 0u};
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int wi = w0 + lane;
    const uint32_t b = wi < words ? bm[wi] : 0u;
    const int c = __popc(b);
    const int incl = warp_incl_scan(c, lane);
    const int tot = __shfl_sync(0xffffffffu, incl, 31);
    if (pos < tot) {
      const int L = __ffs(__ballot_sync(0xffffffffu, incl > pos)) - 1;
      const int ex = __shfl_sync(0xffffffffu, incl - c, L);
      const uint32_t bl = __shfl_sync(0xffffffffu, b, L);
      w.ww = w0 + L;
      w.wrem = drop_low_bits(bl, pos - ex);
      return w;
    }
    pos -= tot;
  }
  return w;
}

// The next kKBlock union rows into ix[0..64) (-1 past the end of the union).
// Four words a step, one bit of each per lane: a set bit's position is the
// rows already placed plus the set bits before it. (A 32-word window with a
// warp scan per block took about 0.5 us a block; one word a step 0.7 us a
// block at a third of the rows: more than the block's copies take.)
__device__ __forceinline__ void walk_block(const uint32_t* bm, int words, UnionWalk& w, int* ix,
                                           int lane) {
  const uint32_t below = (1u << lane) - 1u;
  int filled = 0;
  while (w.ww < words) {
    const int ww = w.ww;
    uint32_t b[4];
    b[0] = w.wrem;
#pragma unroll
    for (int q = 1; q < 4; ++q) b[q] = ww + q < words ? bm[ww + q] : 0u;
    int e[5];  // rows placed before word q
    e[0] = filled;
#pragma unroll
    for (int q = 0; q < 4; ++q) e[q + 1] = e[q] + __popc(b[q]);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int pos = e[q] + __popc(b[q] & below);
      if (((b[q] >> lane) & 1u) && pos < kKBlock) ix[pos] = (ww + q) * 32 + lane;
    }
    if (e[4] >= kKBlock) {
      // the first of the four words that reaches the block's end
      int qs = 3;
#pragma unroll
      for (int q = 2; q >= 0; --q)
        if (e[q + 1] >= kKBlock) qs = q;
      uint32_t bq = b[0];
      int eq = e[0], eq1 = e[1];
#pragma unroll
      for (int q = 1; q < 4; ++q)
        if (q == qs) {
          bq = b[q];
          eq = e[q];
          eq1 = e[q + 1];
        }
      if (eq1 > kKBlock) {  // the word goes on in the next block
        const int pos = eq + __popc(bq & below);
        w.wrem = __ballot_sync(0xffffffffu, ((bq >> lane) & 1u) && pos >= kKBlock);
        w.ww = ww + qs;
      } else {  // the block ends with the word
        w.ww = ww + qs + 1;
        w.wrem = w.ww < words ? bm[w.ww] : 0u;
      }
      return;
    }
    filled = e[4];
    w.ww = ww + 4;
    w.wrem = w.ww < words ? bm[w.ww] : 0u;
  }
  for (int pos = filled + lane; pos < kKBlock; pos += 32) ix[pos] = -1;
}

// 16-byte global -> shared copy; src_bytes 0 fills zeros (nothing is read).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Arrive on bar once this thread's earlier cp.async copies have landed (the
// barrier's count includes these arrivals: one per gather lane).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Two CTAs per SM for decode batches (the host sizes the ring for that), so
// at most 96 registers a thread.
__global__ void __launch_bounds__(kThreads, 2)
    down_tc_kernel(const __grid_constant__ DownTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  const uint32_t stage_bytes = kABytes + p.b_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  uint64_t* empty = full + stages;
  uint64_t* gfull = empty + stages;   // gathered K-block landed (an arrival per gather lane)
  uint64_t* tfull = gfull + stages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* ixfull = drain + 1;          // [kIxSlots] a K-block's union rows are in ixs (warp 0)
  uint64_t* ixempty = ixfull + kIxSlots;  // [kIxSlots] the four gather warps have read them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ixempty + kIxSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_part = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* ixs = reinterpret_cast<int*>(tmem_slot + 4);  // [kIxSlots][kKBlock] union rows
  uint32_t* bm = reinterpret_cast<uint32_t*>(ixs + kIxSlots * kKBlock);  // [fw] union bitmap

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  __shared__ UnitQueue uq;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
      mbar_init(gfull + s, 32 * kGatherWarps);
    }
    for (int i = 0; i < kIxSlots; ++i) {
      mbar_init(ixfull + i, 1);
      mbar_init(ixempty + i, kGatherWarps);
    }
    for (int q = 0; q < kUQ; ++q) {
      mbar_init(&uq.full[q], 1);
      mbar_init(&uq.empty[q], 5 + kGatherWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // TMEM is taken only once the previous kernel has completed, so a CTA of
  // this kernel never holds TMEM while waiting on another kernel
  grid_dep_wait();
  const int n_slices = p.dm.d / kDownSlice;
  const int n_tc = __ldcg(p.ws.meta + kMetaTcCount);
  const int ks = tc_ksplit(p.dm, n_tc);  // > 1: units cut into K parts (ticketed sum)
  const int n_units = n_tc * n_slices * ks;
  if (static_cast<int>(blockIdx.x) >= n_units) return;  // no unit for this CTA: leave before TMEM
  if (warp == 1) tmem_alloc(tmem_slot, p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t buf_cols = p.n_max;

  // Ring stages are used by all-rows K-blocks (full[s], TMA, issued by warp
  // 0) and gathered ones (gfull[s], copies by the gather warps, which take
  // the rows from the union-row slots); every warp sees the same sequence,
  // and keeps one phase bit per stage for each kind (bit s of tbits / gbits).
  if (warp == 0) {
    // ------------------------------------------------ TMA producer / union walk
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_wd_blk);
      tma_prefetch_desc(&p.tm_wds_blk);
      tma_prefetch_desc(&p.tm_ht_blk);
    }
    uint32_t it = 0, gi = 0, tbits = 0, tlast = 0;
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int u =
          uq_take(uq, n, p.ws.meta + kMetaTcQueue, n_units, abort_flag, p.ws.status, lane);
      if (u == -2) ok = false;
      if (u < 0) break;
      const DownUnit du = decode(p, u, n_slices, ks);
      if (du.slice == 0 && du.part == 0 && lane == 0) {
        if (du.cand && !du.skip) {  // a candidate taken here
          atomicAdd(p.ws.counters + kCntDownRows, static_cast<unsigned long long>(du.F_e));
          atomicAdd(p.ws.counters + kCntTc, 1ull);
        }
        if (du.auto_gather) {  // the router counted all rows: count the union instead
          atomicAdd(p.ws.counters + kCntDownRows,
                    static_cast<unsigned long long>(static_cast<long long>(du.cnt - du.F_e)));
          atomicAdd(p.ws.counters + kCntTcGather, 1ull);
        }
      }
      const int N = (du.gr.m + 15) & ~15;
      const int x0 = du.slice * kDownSlice;
      const CUtensorMap* wblk = du.shared ? &p.tm_wds_blk : &p.tm_wd_blk;
      const int words = du.F_e / 32;
      UnionWalk wk{0, 0u};
      if (du.gather && du.nk > 0) {
        // the group's union bitmap into shared memory (the previous unit's
        // walk is over), then the walk position of this part's first row
        __syncwarp();
        const uint32_t* bits = p.ws.union_bits + static_cast<size_t>(du.g) * p.dm.fw;
        for (int i0 = 0; i0 < words; i0 += 4 * 32) {  // four loads in flight a lane
          uint32_t v[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = i0 + 32 * q + lane;
            v[q] = i < words ? __ldcg(bits + i) : 0u;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (i0 + 32 * q + lane < words) bm[i0 + 32 * q + lane] = v[q];
        }
        __syncwarp();
        wk = walk_seek(bm, words, du.k0 * kKBlock, lane);
      }
      for (int kc = du.k0; kc < du.k0 + du.nk; ++kc, ++it) {
        const uint32_t s = it % stages;
        if (du.gather) {
          // the next union-row slot, once the gather warps have read it
          const uint32_t x = gi % kIxSlots;
          if (!warp_wait(ixempty + x, ((gi / kIxSlots) & 1u) ^ 1u, abort_flag, p.ws.status)) {
            ok = false;
            break;
          }
          walk_block(bm, words, wk, ixs + x * kKBlock, lane);
          __syncwarp();
          if (lane == 0) mbar_arrive(ixfull + x);  // release: the rows are visible to the gather warps
          ++gi;
        } else {
          const uint32_t ph = (it / stages) & 1u;
          if (!warp_wait(empty + s, ph ^ 1u, abort_flag, p.ws.status)) { ok = false; break; }
          uint8_t* sa = smem + s * stage_bytes;
          const int nb = (N + 63) / 64;
          if (lane == 0) {
            mbar_arrive_expect_tx(full + s, kABytes + nb * 64 * 128);
            const int wy = du.row_base + kc * kKBlock;
            tma_load_2d(sa, wblk, full + s, x0, wy);
            tma_load_2d(sa + kAAtom, wblk, full + s, x0 + 64, wy);
          }
          __syncwarp();
          if (lane < nb)
            tma_load_2d(sa + kABytes + lane * kAAtom, &p.tm_ht_blk, full + s,
                        du.gr.slot0 + 64 * lane, kc * kKBlock);
          tbits ^= 1u << s;
          tlast |= 1u << s;
        }
        __syncwarp();
      }
    }
    // the TMA copies still in flight land before the CTA can leave (the
    // gather warps wait for their own copies)
    if (lane == 0) {
      volatile int never = 0;
      for (int s = 0; s < stages; ++s)
        if ((tlast >> s) & 1u) mbar_wait(full + s, ((tbits >> s) & 1u) ^ 1u, &never, p.ws.status);
    }
    __syncwarp();
  } else if (warp >= kGatherWarp0) {
    // ------------------------------------------------ gather copies (warps 6..9)
    const int gw = warp - kGatherWarp0;
    const uint32_t ht_ld = static_cast<uint32_t>(p.dm.slots_total);
    uint32_t it = 0, gi = 0;
    for (int n = 0;; ++n) {
      const int u = uq_next(uq, n, abort_flag, p.ws.status, lane);
      if (u < 0) break;
      const DownUnit du = decode(p, u, n_slices, ks);
      if (!du.gather) {
        it += du.nk;
        continue;
      }
      const int N = (du.gr.m + 15) & ~15;
      const int x0 = du.slice * kDownSlice;
      const __nv_bfloat16* wsrc = static_cast<const __nv_bfloat16*>(du.shared ? p.wds : p.wd) +
                                  static_cast<size_t>(du.row_base) * p.dm.d + x0;
      const __nv_bfloat16* hsrc = static_cast<const __nv_bfloat16*>(p.ht) + du.gr.slot0;
      // B chunks (8 slots each) that exist: the MMA reads N slots; slots past
      // the end of H^T are zero-filled
      const int hchunks = N / 8;
      const int hlim = static_cast<int>(ht_ld) - du.gr.slot0;
      bool ok = true;
      for (int kc = 0; kc < du.nk; ++kc, ++it, ++gi) {
        const uint32_t s = it % stages;
        const uint32_t x = gi % kIxSlots;
        // the K-block's union rows (into registers first), then its ring
        // stage free; the waits on the MMA poll tightly (each probe may
        // suspend the thread in hardware until the phase completes)
        if (!warp_wait(ixfull + x, (gi / kIxSlots) & 1u, abort_flag, p.ws.status)) {
          ok = false;
          break;
        }
        const int* ix = ixs + x * kKBlock + gw * kGatherRows;
        int ja[kGatherRows / 2], jb[kGatherRows / 4];
#pragma unroll
        for (int i = 0; i < kGatherRows / 2; ++i) ja[i] = ix[2 * i + (lane >> 4)];
#pragma unroll
        for (int i = 0; i < kGatherRows / 4; ++i) jb[i] = ix[4 * i + (lane >> 3)];
        if (!warp_wait(empty + s, ((it / stages) & 1u) ^ 1u, abort_flag, p.ws.status, 32)) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_u32(smem + s * stage_bytes);
        // A: 16 rows x 16 chunks of 16 B; lanes 0-15 one row, 16-31 the next
        const int c = lane & 15;
#pragma unroll
        for (int i = 0; i < kGatherRows / 2; ++i) {
          const int q = 2 * i + (lane >> 4);
          const int j = ja[i];
          const int r = gw * kGatherRows + q;  // packed K position
          const uint32_t dst =
              sa + (c >> 3) * kAAtom + r * 128 + ((((c & 7) ^ (r & 7))) << 4);
          cp_async16(dst, wsrc + static_cast<size_t>(j < 0 ? 0 : j) * p.dm.d + c * 8,
                     j < 0 ? 0u : 16u);
        }
        // B: 16 rows x 8 chunks of 16 B (8 slots); lanes 8 q .. 8 q + 7 one row
        const int cb = lane & 7;
#pragma unroll
        for (int i = 0; i < kGatherRows / 4; ++i) {
          const int q = 4 * i + (lane >> 3);
          const int j = jb[i];
          const int r = gw * kGatherRows + q;
          const uint32_t dst = sa + kABytes + r * 128 + ((cb ^ (r & 7)) << 4);
          const bool has = j >= 0 && cb < hchunks && 8 * cb + 8 <= hlim;
          cp_async16(dst, hsrc + static_cast<size_t>(has ? j : 0) * ht_ld + (has ? 8 * cb : 0),
                     has ? 16u : 0u);
        }
        cp_async_arrive(gfull + s);
        __syncwarp();
        if (lane == 0) mbar_arrive(ixempty + x);  // this warp's rows of the slot are read
      }
      if (!ok) break;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    uint32_t it = 0, uidx = 0, tbits = 0, gbits = 0;
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int u = uq_next(uq, n, abort_flag, p.ws.status, lane);
      if (u < 0) break;
      const DownUnit du = decode(p, u, n_slices, ks);
      if (du.nk == 0) continue;  // empty union: the epilogue writes zeros
      const int N = (du.gr.m + 15) & ~15;
      const uint32_t idesc = idesc_bf16_f32(kDownSlice, N, 1, 1);
      const uint32_t b = uidx % 2;
      const uint32_t tph = (uidx / 2) & 1u;
      if (!warp_wait(tempty + b, tph ^ 1u, abort_flag, p.ws.status)) break;
      tc_fence_after();
      const uint32_t d_t = tmem_base + b * buf_cols;
      for (int kc = 0; kc < du.nk; ++kc, ++it) {
        const uint32_t s = it % stages;
        if (du.gather) {
          if (!warp_wait(gfull + s, (gbits >> s) & 1u, abort_flag, p.ws.status, 32)) {
            ok = false;
            break;
          }
          gbits ^= 1u << s;
          // the gather copies are generic-proxy writes; the MMA reads shared
          // memory through the async proxy
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        } else {
          if (!warp_wait(full + s, (tbits >> s) & 1u, abort_flag, p.ws.status)) {
            ok = false;
            break;
          }
          tbits ^= 1u << s;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sa = smem_u32(smem + s * stage_bytes);
          const uint64_t ad = smem_desc_sw128(sa, kAAtom, 1024);
          const uint64_t bd = smem_desc_sw128(sa + kABytes, kAAtom, 1024);
#pragma unroll
          for (int kk = 0; kk < kKBlock / 16; ++kk) {
            // 16 K-rows of 128 B per step = 2048 B (descriptor units of 16 B)
            mma_bf16(d_t, ad + 128 * kk, bd + 128 * kk, idesc, (kc | kk) != 0);
          }
          mma_commit(empty + s);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) mma_commit(tfull + b);
      __syncwarp();
      ++uidx;
    }
    if (lane == 0) {
      mma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never, p.ws.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const int d = p.dm.d;
    uint32_t uidx = 0;
    for (int n = 0;; ++n) {
      const int u = uq_next(uq, n, abort_flag, p.ws.status, lane);
      // the four warps leave together (the part path below has barriers)
      const bool got = ks > 1 ? epi_all(u != -2) : u != -2;
      if (!got || u < 0) break;
      const DownUnit du = decode(p, u, n_slices, ks);
      const int m = du.gr.m;
      const int col = du.slice * kDownSlice + 32 * q + lane;
      float* yc = p.ws.y + static_cast<size_t>(du.gr.slot0) * d + col;
      if (du.skip) continue;  // the GEMV kernel has added this group's rows into Y
      // parts: this part's sums go to its block of the part buffer, [token][128 columns]
      float* pc = p.ws.tc_part +
                  (static_cast<size_t>(du.ub) * ks + du.part) * kTcPartTokens * kDownSlice + 32 * q +
                  lane;
      if (du.nk == 0) {
        // no K-blocks (an empty union, or a part of a small gathered union):
        // zeros, as the unit's sums or as this part's
        if (ks == 1) {
          for (int c = 0; c < m; ++c) yc[static_cast<size_t>(c) * d] = 0.f;
          continue;
        }
        for (int c = 0; c < m; ++c) pc[c * kDownSlice] = 0.f;
      } else {
        const int N = (m + 15) & ~15;
        const uint32_t b = uidx % 2;
        const uint32_t tph = (uidx / 2) & 1u;
        bool ok = warp_wait(tfull + b, tph, abort_flag, p.ws.status);
        if (ks > 1) ok = epi_all(ok);  // the part path's barriers below need all four warps
        if (!ok) break;
        tc_fence_after();
        const uint32_t ta = tmem_base + lane_off + b * buf_cols;
        for (int c0 = 0; c0 < N; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(ta + c0, r);
          tmem_ld_wait(r);
          if (ks == 1) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c0 + i < m) yc[static_cast<size_t>(c0 + i) * d] = __uint_as_float(r[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c0 + i < m) pc[(c0 + i) * kDownSlice] = __uint_as_float(r[i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty + b);
        ++uidx;
      }
      if (ks > 1) {
        // the last part of this (group, slice) to finish adds the ks parts
        // in part order and stores Y
        const int ub = du.ub;
        __threadfence();
        epi_bar();  // the four warps' columns of this part are written
        if (warp == 2 && lane == 0) *last_part = atomicAdd(p.ws.tc_ticket + ub, 1) == ks - 1;
        epi_bar();
        if (*last_part) {
          __threadfence();
          const float* pb = p.ws.tc_part + static_cast<size_t>(ub) * ks * kTcPartTokens * kDownSlice +
                            32 * q + lane;
          // 8 tokens x 4 parts per batch: their loads are in flight together
          // (one L2 round trip per batch, not one per value); the sums run
          // in part order
          constexpr int kC = 8, kP = 4;
          for (int c0 = 0; c0 < m; c0 += kC) {
            float acc[kC];
#pragma unroll
            for (int i = 0; i < kC; ++i) acc[i] = 0.f;
            for (int p0 = 0; p0 < ks; p0 += kP) {
              float v[kC][kP];
#pragma unroll
              for (int i = 0; i < kC; ++i)
#pragma unroll
                for (int pp = 0; pp < kP; ++pp)
                  v[i][pp] = c0 + i < m && p0 + pp < ks
                                 ? __ldcg(pb + (static_cast<size_t>(p0 + pp) * kTcPartTokens +
                                                c0 + i) *
                                                   kDownSlice)
                                 : 0.f;
#pragma unroll
              for (int i = 0; i < kC; ++i)
#pragma unroll
                for (int pp = 0; pp < kP; ++pp) acc[i] += v[i][pp];
            }
#pragma unroll
            for (int i = 0; i < kC; ++i)
              if (c0 + i < m) yc[static_cast<size_t>(c0 + i) * d] = acc[i];
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace

size_t down_tc_smem_bytes(int b_bytes, int stages, int fw) {
  return 1024 + static_cast<size_t>(stages) * (kABytes + b_bytes) +
         (3 * stages + 5 + 2 * kIxSlots) * sizeof(uint64_t) + 16 +
         static_cast<size_t>(kIxSlots) * kKBlock * 4 + static_cast<size_t>(fw) * 4;
}

cudaError_t launch_down_tc(const DownTcParams& p, int grid, size_t smem, cudaStream_t st) {
  // the limit covers this launch's dynamic shared memory (the kernel also
  // has a little static shared memory, so 227 KB of dynamic would not fit)
  const cudaError_t e = smem_limit(down_tc_kernel, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(down_tc_kernel, grid, kThreads, smem, st, p);
}

}  // namespace moe
