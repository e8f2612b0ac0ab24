// Consumer-side arithmetic of the row-streaming kernels: the down
// projection's accumulate-and-flush (Rows) and the sparse up projection's
// partial dot products (UpDots), for bf16 (tensor cores, mma.sync) and fp32
// (packed fp32x2 FMAs) rows.
#pragma once

#include "gemv_common.cuh"

namespace moe {
namespace {

constexpr int kTok = 8;         // token columns of the mma (passes hold up to 8)
constexpr int kTokStride = kTok;  // floats per row of an fp32 h array [row][token]
constexpr int kHBytes = 32;          // h bytes per row slot: 8 x bf16 (16 B used) or 8 x fp32

// TILES: 16-column tiles of a consumer warp's slice (bf16: 16 for a
// 512-byte slice, 32 for 1 KB); the fp32 rows take 512-byte slices.
template <typename TW, int TILES = 16>
struct Rows;

// bf16: tensor-core multiply of the landed rows.
template <int TILES>
struct Rows<__nv_bfloat16, TILES> {
  static constexpr int MT = kGemvTokens;  // tokens per pass
  static constexpr int kTiles = TILES;    // 16-column tiles of the warp's slice
  float acc[kTiles][4];

  __device__ void zero() {
#pragma unroll
    for (int i = 0; i < kTiles; ++i)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[i][v] = 0.f;
  }
  // D[16 columns][8 tokens] += W^T[16 columns][8 rows] * H[8 rows][8 tokens];
  // tokens >= mt and rows >= cnt enter as zero h. h from the stage's bf16 h
  // slots (hs) ...
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
    mma_rows(rows_s, stride, hb2, lane);
  }
  // ... or from fp32 values hf[row][kTokStride], rounded to bf16 (RNE)
  __device__ void consume_hf(uint32_t rows_s, const uint8_t*, int stride, const float* hf, int cnt,
                             int mt, int lane) {
    const int g = lane >> 2, c2 = 2 * (lane & 3);
    uint32_t hb2 = 0u;
    if (g < mt) {
      const float lo = c2 < cnt ? hf[c2 * kTokStride + g] : 0.f;
      const float hi = c2 + 1 < cnt ? hf[(c2 + 1) * kTokStride + g] : 0.f;
      __nv_bfloat162 v2 = __floats2bfloat162_rn(lo, hi);
      hb2 = *reinterpret_cast<uint32_t*>(&v2);
    }
    mma_rows(rows_s, stride, hb2, lane);
  }
  __device__ void mma_rows(uint32_t rows_s, int stride, uint32_t hb2, int lane) {
    const uint32_t row_s = rows_s + (lane & 7) * stride + (lane >> 3) * 16;
#pragma unroll
    for (int p = 0; p < kTiles / 2; ++p) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(row_s + p * 64, a0, a1, a2, a3);
      mma_16x8x8(acc[2 * p], a0, a1, hb2);
      mma_16x8x8(acc[2 * p + 1], a2, a3, hb2);
    }
  }
  // acc[i] = D[column 16i + g (+8)][tokens c2, c2 + 1]: lanes g and g ^ 1
  // swap halves so that each holds two adjacent columns of one token, added
  // into Y with 8-byte vector atomics (no shared-memory staging, so the ring
  // of stages gets that space).
  __device__ void flush(float* y, int d, int mt, int lane) {
    const int tok = 2 * (lane & 3) + ((lane >> 2) & 1);
    flush_to(y + (size_t)tok * d, 1.f, tok < mt, lane);
  }
  // The token of this lane in the flush (its sums go to that token's row).
  __device__ static int flush_token(int lane) { return 2 * (lane & 3) + ((lane >> 2) & 1); }
  // Adds w x the sums of this lane's token (flush_token) into the row yrow
  // (at the warp's first column); nothing when !on.
  __device__ void flush_to(float* yrow, float w, bool on, int lane) {
    const int g = lane >> 2;
    const bool odd = g & 1;
    float* yt = yrow + (g & ~1);
#pragma unroll
    for (int i = 0; i < kTiles; ++i) {
      const float s0 = odd ? acc[i][0] : acc[i][1];
      const float s1 = odd ? acc[i][2] : acc[i][3];
      const float r0 = __shfl_xor_sync(0xffffffffu, s0, 4);
      const float r1 = __shfl_xor_sync(0xffffffffu, s1, 4);
      if (on) {
        const float2 a = odd ? make_float2(r0, acc[i][1]) : make_float2(acc[i][0], r0);
        const float2 b = odd ? make_float2(r1, acc[i][3]) : make_float2(acc[i][2], r1);
        red_add_v2(yt + 16 * i, w * a.x, w * a.y);
        red_add_v2(yt + 16 * i + 8, w * b.x, w * b.y);
      }
    }
  }
};

// fp32: packed fp32x2 FMAs, 4 columns per lane, up to 8 tokens.
template <int TILES>
struct Rows<float, TILES> {
  static constexpr int MT = 8;
  uint64_t acc[MT][2];

  __device__ void zero() {
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = 0ull;
  }
  __device__ void consume_hf(uint32_t, const uint8_t* rows, int stride, const float* hf, int cnt,
                             int mt, int lane) {
    for (int r = 0; r < cnt; ++r) fma_row(rows + r * stride, hf + r * kTokStride, mt, lane);
  }
  __device__ void fma_row(const uint8_t* wrow, const float* hr, int mt, int lane) {
    const uint4 u = *reinterpret_cast<const uint4*>(wrow + lane * 16);
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
  __device__ void flush(float* y, int d, int mt, int lane) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t < mt) {
        const float2 a = unpack2(acc[t][0]), b = unpack2(acc[t][1]);
        red_add_v4(y + (size_t)t * d + lane * 4, a.x, a.y, b.x, b.y);
      }
    }
  }
  // Adds w[t] x the sums of token t into the row yrow[t] (at the warp's
  // first column) for t < mt.
  __device__ void flush_rows(float* const (&yrow)[MT], const float (&w)[MT], int mt, int lane) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      if (t < mt) {
        const float2 a = unpack2(acc[t][0]), b = unpack2(acc[t][1]);
        red_add_v4(yrow[t] + lane * 4, w[t] * a.x, w[t] * a.y, w[t] * b.x, w[t] * b.y);
      }
    }
  }
};

// d += A (16 x 16, bf16) * B (16 x 8, bf16), fp32 accumulation, all 16 rows.
__device__ __forceinline__ void mma_16x8x16_a4(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Four 8x8 bf16 matrices from shared memory (every lane supplies a row address).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                       uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

template <typename TW>
struct UpDots;

// bf16: 16 K-steps of 16 columns over the warp's 256 columns, 16 rows a
// stage (the mma's M).
template <>
struct UpDots<__nv_bfloat16> {
  static constexpr int MT = kGemvTokens;
  static constexpr int kRows = 16;   // rows per stage
  static constexpr int kParts = 4;   // partial dots per lane and stage
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
  // partial dots of the stage's 16 rows over this warp's slice: p[0..1] =
  // (row g, tokens c2, c2 + 1), p[2..3] = (row g + 8, the same tokens)
  __device__ void dots(uint32_t rows_s, const uint8_t*, int stride, float (&p)[kParts], int lane) {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    // ldmatrix x4: lanes 0-7 rows 0-7 and lanes 8-15 rows 8-15 at the K-step's
    // first 8 columns, lanes 16-31 the same rows at its last 8
    const uint32_t a_addr =
        rows_s + ((lane & 7) + ((lane >> 3) & 1) * 8) * stride + (lane >> 4) * 16;
#pragma unroll
    for (int ks = 0; ks < 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(a_addr + 32 * ks, a0, a1, a2, a3);
      mma_16x8x16_a4(d, a0, a1, a2, a3, xb[ks][0], xb[ks][1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = d[i];
  }
  // where this lane's partials go: (row, token) pairs
  __device__ static void owner(int lane, int i, int& row, int& tok) {
    row = (lane >> 2) + 8 * (i >> 1);
    tok = 2 * (lane & 3) + (i & 1);
  }
};

// fp32: 4 columns per lane, warp reduction per (row, token), 8 rows a stage.
template <>
struct UpDots<float> {
  static constexpr int MT = 8;
  static constexpr int kRows = 8;
  static constexpr int kParts = 2;
  float xv[MT][4];

  __device__ void load_x(const float* xrows, int d, int mt, int col0, int lane) {
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        xv[t][i] = t < mt ? __ldcg(xrows + (size_t)t * d + col0 + 4 * lane + i) : 0.f;
  }
  __device__ void dots(uint32_t, const uint8_t* rows, int stride, float (&p)[kParts], int lane) {
    // 64 (row, token) sums; lane l ends with those of (row l / 8, tokens ..)
    p[0] = p[1] = 0.f;
#pragma unroll 1
    for (int r = 0; r < kRows; ++r) {
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

}  // namespace
}  // namespace moe
