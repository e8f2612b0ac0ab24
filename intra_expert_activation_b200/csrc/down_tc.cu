// Down projection on the 5th-generation tensor cores, reading only the
// W_down rows of an expert token group's active-neuron union.
//
// The pages' kernel gathers the weights of the active neurons, packs them
// densely in shared memory and multiplies densely [gist.science EN
// "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
// Model Execution", Technical Summary > Methodology > System Implementation in
// vLLM > "Fused Up-Down Projection"]. Here the packing is done by TMA: four
// active rows per copy (tile::gather4 over a tensor map whose box is one row,
// 128-byte swizzled) land at their packed positions, so the tensor core sees
// a dense K-block of union rows.
//
// Work unit: (group, 128-column slice of d_model); K = the group's union rows.
//   D[128 columns][N tokens] = W_down[e][U, slice]^T . H^T[U, group slots]
// Both operands are MN-major in shared memory: a W_down row is 128
// contiguous output columns (M), an H^T row is 64 contiguous slots (N).
//   gathered mode: K-block = 64 union rows, four per gather4 copy (A: two
//     copies of 64 columns, B: one of 64 slots, per four rows); in the last
//     K-block of a unit the positions past the union repeat the last union
//     row of W_down and fetch H^T rows out of range one by one (zeros).
//   all-rows mode: K-block = 64 consecutive rows with 64-row boxes; h of
//     inactive neurons is an exact zero, so the sum is the same.
// Warp roles as in the gate/up kernel: warp 0 TMA, warp 1 MMA + TMEM owner,
// warps 2-5 drain TMEM into Y[slot][col] (fp32), coalesced across lanes.
// With few units for the grid (decode batches with one to a few groups on
// this path), a unit's K-blocks are cut into parts (tc_ksplit): each part
// drains its sums into a workspace block, and the part that finishes last
// (an atomic ticket per unit) adds the parts in part order and stores Y.
// A candidate group that the row stream takes (cand_takes_gemv) is skipped.
#include "common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 192;

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
  uint64_t empty[kUQ];         // the MMA warp and the 4 epilogue warps read it (5 arrivals)
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
  du.gather = path == kPathTcGather;
  du.cnt = __ldcg(p.ws.union_cnt + du.g);
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

__global__ void __launch_bounds__(kThreads, 1)
    down_tc_kernel(const __grid_constant__ DownTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  const uint32_t stage_bytes = kABytes + p.b_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  uint64_t* empty = full + stages;
  uint64_t* tfull = empty + stages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_part = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  __shared__ UnitQueue uq;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int q = 0; q < kUQ; ++q) {
      mbar_init(&uq.full[q], 1);
      mbar_init(&uq.empty[q], 5);
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
  const int ht_oob = p.dm.F_max;  // H^T row past the end: zero fill

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_wd_row);
      tma_prefetch_desc(&p.tm_wd_blk);
      tma_prefetch_desc(&p.tm_ht_row);
      tma_prefetch_desc(&p.tm_ht_blk);
    }
    uint32_t it = 0;
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int u =
          uq_take(uq, n, p.ws.meta + kMetaTcQueue, n_units, abort_flag, p.ws.status, lane);
      if (u == -2) ok = false;
      if (u < 0) break;
      const DownUnit du = decode(p, u, n_slices, ks);
      if (du.cand && !du.skip && du.slice == 0 && du.k0 == 0 && lane == 0) {  // a candidate taken here
        atomicAdd(p.ws.counters + kCntDownRows,
                  static_cast<unsigned long long>(du.shared ? p.dm.Fs : p.dm.F));
        atomicAdd(p.ws.counters + kCntTc, 1ull);
      }
      const int N = (du.gr.m + 15) & ~15;
      const int x0 = du.slice * kDownSlice;
      const int* rows = p.ws.union_rows + static_cast<size_t>(du.g) * p.dm.F_max;
      const CUtensorMap* wrow = du.shared ? &p.tm_wds_row : &p.tm_wd_row;
      const CUtensorMap* wblk = du.shared ? &p.tm_wds_blk : &p.tm_wd_blk;
      for (int kc = du.k0; kc < du.k0 + du.nk; ++kc, ++it) {
        const uint32_t s = it % stages;
        const uint32_t ph = (it / stages) & 1u;
        if (!warp_wait(empty + s, ph ^ 1u, abort_flag, p.ws.status)) { ok = false; break; }
        uint8_t* sa = smem + s * stage_bytes;
        uint8_t* sb = sa + kABytes;
        if (du.gather) {
          // four union rows per copy (tile::gather4, boxes one row high): lane
          // l < 16 fetches packed positions 4 l .. 4 l + 3 of the K-block. Past
          // the union the W_down rows repeat the last union row (inside the
          // tensor) and the H^T rows are fetched out of range one by one, which
          // fills zeros, so those positions add nothing
          if (lane == 0) mbar_arrive_expect_tx(full + s, kABytes + 64 * 128);
          __syncwarp();
          const int base = kc * kKBlock;
          const bool whole_blk = base + kKBlock <= du.cnt;
          if (lane < 16) {
            int jr[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              jr[q] = __ldcg(rows + min(base + 4 * lane + q, du.cnt - 1));
            tma_gather4_2d(sa + lane * 512, wrow, full + s, x0, du.row_base + jr[0],
                           du.row_base + jr[1], du.row_base + jr[2], du.row_base + jr[3]);
            tma_gather4_2d(sa + kAAtom + lane * 512, wrow, full + s, x0 + 64, du.row_base + jr[0],
                           du.row_base + jr[1], du.row_base + jr[2], du.row_base + jr[3]);
            if (whole_blk)
              tma_gather4_2d(sb + lane * 512, &p.tm_ht_row, full + s, du.gr.slot0, jr[0], jr[1],
                             jr[2], jr[3]);
          }
          if (!whole_blk) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int r = lane + 32 * h;
              const int pos = base + r;
              const int hy = pos < du.cnt ? __ldcg(rows + pos) : ht_oob;
              tma_load_2d(sb + r * 128, &p.tm_ht_row, full + s, du.gr.slot0, hy);
            }
          }
        } else {
          const int nb = (N + 63) / 64;
          if (lane == 0) {
            mbar_arrive_expect_tx(full + s, kABytes + nb * 64 * 128);
            const int wy = du.row_base + kc * kKBlock;
            tma_load_2d(sa, wblk, full + s, x0, wy);
            tma_load_2d(sa + kAAtom, wblk, full + s, x0 + 64, wy);
          }
          __syncwarp();
          if (lane < nb)
            tma_load_2d(sb + lane * kAAtom, &p.tm_ht_blk, full + s, du.gr.slot0 + 64 * lane,
                        kc * kKBlock);
        }
        __syncwarp();
      }
    }
    const uint32_t n_tail = it < (uint32_t)stages ? it : (uint32_t)stages;
    if (lane == 0) {
      volatile int never = 0;
      for (uint32_t i = it - n_tail; i < it; ++i)
        mbar_wait(full + (i % stages), (i / stages) & 1u, &never, p.ws.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    uint32_t it = 0, uidx = 0;
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
        const uint32_t ph = (it / stages) & 1u;
        if (!warp_wait(full + s, ph, abort_flag, p.ws.status)) { ok = false; break; }
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
      if (du.nk == 0) {  // empty union (gathered mode, never cut into parts)
        for (int c = 0; c < m; ++c) yc[static_cast<size_t>(c) * d] = 0.f;
        continue;
      }
      const int N = (m + 15) & ~15;
      const uint32_t b = uidx % 2;
      const uint32_t tph = (uidx / 2) & 1u;
      bool ok = warp_wait(tfull + b, tph, abort_flag, p.ws.status);
      if (ks > 1) ok = epi_all(ok);  // the part path's barriers below need all four warps
      if (!ok) break;
      tc_fence_after();
      // parts: this part's sums go to its block of the part buffer, [token][128 columns]
      float* pc = p.ws.tc_part +
                  (static_cast<size_t>(du.ub) * ks + du.part) * kTcPartTokens * kDownSlice + 32 * q +
                  lane;
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
          // 8 tokens x 6 parts per batch: their loads are in flight together
          // (one L2 round trip per batch, not one per value); the sums run
          // in part order
          constexpr int kC = 8, kP = 6;
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

size_t down_tc_smem_bytes(int b_bytes, int stages) {
  return 1024 + static_cast<size_t>(stages) * (kABytes + b_bytes) +
         (2 * stages + 5) * sizeof(uint64_t) + 16;
}

cudaError_t launch_down_tc(const DownTcParams& p, int grid, size_t smem, cudaStream_t st) {
  // the limit covers this launch's dynamic shared memory (the kernel also
  // has a little static shared memory, so 227 KB of dynamic would not fit)
  const cudaError_t e = smem_limit(down_tc_kernel, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(down_tc_kernel, grid, kThreads, smem, st, p);
}

}  // namespace moe
