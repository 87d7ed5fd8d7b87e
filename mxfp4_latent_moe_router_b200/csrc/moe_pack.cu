// moe_pack.cu -- one-time repacking of canonical weights into MMA-fragment tiles.
//
// Canonical inputs (see include/moe.h): bf16 tensors in "x . W" orientation
// [K][N]; MXFP4 tensors output-row-major [rows][K/2] codes + [rows][K/32]
// e8m0 scales.  Outputs are the tile layouts described in layout.cuh.
#include <cuda_runtime.h>

#include "engine.cuh"
#include "layout.cuh"

namespace moe {

// dense layouts
enum : int { DENSE_PLAIN = 0, DENSE_GATE_UP = 1, DENSE_TWO_K = 2 };
// MXFP4 layouts
enum : int { MX_PLAIN = 0, MX_GATE_UP = 1 };

// Unit u of a tile is 16 bytes: 8 bf16 values.  Warp-MMA order: lane, k16
// step, 32-block and warp tile of the m16n8k16 A fragments.  Tensor-core
// order (umma): core-matrix slot u = (kb * 16 + rg) * 8 + rr holds row
// 8 rg + rr, K elements 8 kb .. 8 kb + 7 of the chunk (row groups 128 bytes
// apart, K blocks 2048).  Either way a row of the tile is row r of warp tile
// w (16 rows each), as the epilogues expect.
__global__ void pack_dense_kernel(const uint16_t* __restrict__ src, int K, int N, int layout,
                                  int RB, int C, uint8_t* __restrict__ dst,
                                  const uint16_t* __restrict__ src2, int K2, int C_first, int umma) {
  const long long units = (long long)RB * C * 1024;
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < units;
       u += (long long)gridDim.x * blockDim.x) {
    const int lane = u & 31, s = (u >> 5) & 1, b = (u >> 6) & 1, w0 = (u >> 7) & 7;
    const long long tile = u >> 10;
    const int rb = (int)(tile / C), c = (int)(tile % C);
    const int g = lane >> 2, t = lane & 3;
    const int slot = (int)(u & 1023);
    uint16_t v[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        int w = w0, r, kk;
        if (umma) {
          const int row = ((slot >> 3) & 15) * 8 + (slot & 7);  // row within the tile
          w = row >> 4;
          r = row & 15;
          kk = 8 * (slot >> 7) + 2 * q + e;
        } else {
          r = frag_row(g, q);  // row within the warp tile
          kk = 32 * b + frag_k(t, s, q, e);
        }
        const uint16_t* m = src;
        int col = -1, k = -1, kmax = K;
        if (layout == DENSE_PLAIN) {
          col = rb * kRowsPerBlock + 16 * w + r;
          k = c * kDenseChunkK + kk;
        } else if (layout == DENSE_GATE_UP) {
          col = 64 * rb + 8 * w + (r & 7);
          if (r >= 8) m = src2;
          k = c * kDenseChunkK + kk;
        } else {  // DENSE_TWO_K: rows = output columns n, K = [src rows ; src2 rows]
          col = rb * kRowsPerBlock + 16 * w + r;
          if (c < C_first) {
            k = c * kDenseChunkK + kk;
          } else {
            m = src2;
            kmax = K2;
            k = (c - C_first) * kDenseChunkK + kk;
          }
        }
        uint16_t val = 0;
        if (col < N && k < kmax) val = m[(long long)k * N + col];
        v[2 * q + e] = val;
      }
    }
    uint4 o;
    o.x = v[0] | ((uint32_t)v[1] << 16);
    o.y = v[2] | ((uint32_t)v[3] << 16);
    o.z = v[4] | ((uint32_t)v[5] << 16);
    o.w = v[6] | ((uint32_t)v[7] << 16);
    // [warp][blk][step][lane][16 B], or the core-matrix slot
    uint8_t* d = dst + tile * kDenseTileBytes +
                 (umma ? slot * 16 : (((w0 * 2 + b) * 2 + s) * 32 + lane) * 16);
    *reinterpret_cast<uint4*>(d) = o;
  }
}

__device__ __forceinline__ int mx_src_row(int layout, int rb, int row_in_block, int rows_half,
                                          int rows, bool& valid) {
  if (layout == MX_GATE_UP) {
    const int w = row_in_block >> 4, r = row_in_block & 15;
    const int h = 64 * rb + 8 * w + (r & 7);  // SwiGLU output index
    valid = h < rows_half;
    return (r < 8) ? h : rows_half + h;
  }
  const int row = rb * kRowsPerBlock + row_in_block;
  valid = row < rows;
  return row;
}

// The tensor-core tile order (layout.cuh): unit v < 1024 is code slot v (16
// bytes: 32 K elements of one row), unit 1024 + i the scale bytes 16 i ..
// 16 i + 15.
__device__ __forceinline__ void pack_mx_umma_unit(const uint8_t* ce, const uint8_t* se, int layout,
                                                  int rb, int c, int rows, int rows_half, int K,
                                                  int v, uint8_t* tdst, int* err) {
  const int kb_total = K / 32;
  uint8_t out[16];
  if (v < 1024) {
    const int r = v & 7, rg = (v >> 3) & 15, kb = v >> 7;
    bool valid;
    const int sr = mx_src_row(layout, rb, rg * 8 + r, rows_half, rows, valid);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int k = c * kMxChunkK + kb * 32 + 2 * j;
      out[j] = (valid && k < K) ? ce[(long long)sr * (K / 2) + k / 2] : 0;
    }
    uint4 o;
    o.x = out[0] | (out[1] << 8) | (out[2] << 16) | ((uint32_t)out[3] << 24);
    o.y = out[4] | (out[5] << 8) | (out[6] << 16) | ((uint32_t)out[7] << 24);
    o.z = out[8] | (out[9] << 8) | (out[10] << 16) | ((uint32_t)out[11] << 24);
    o.w = out[12] | (out[13] << 8) | (out[14] << 16) | ((uint32_t)out[15] << 24);
    *reinterpret_cast<uint4*>(tdst + v * 16) = o;
    return;
  }
  const int o0 = (v - 1024) * 16;  // byte offset in the two 512-byte units
  const int unit = o0 >> 9, m0 = (o0 & 511) >> 4;
  int bad = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int m = m0 + 32 * (j >> 2), kb = 4 * unit + (j & 3);
    const int blk = c * 8 + kb;
    bool valid;
    const int sr = mx_src_row(layout, rb, m, rows_half, rows, valid);
    uint8_t sv = 127;
    if (valid && blk < kb_total) {
      sv = se[(long long)sr * kb_total + blk];
      if (sv == 0xFF) bad = 1;
    }
    out[j] = sv;
  }
  if (bad) atomicOr(err, 1 << ERR_NAN_SCALE);
  uint4 o;
  o.x = out[0] | (out[1] << 8) | (out[2] << 16) | ((uint32_t)out[3] << 24);
  o.y = out[4] | (out[5] << 8) | (out[6] << 16) | ((uint32_t)out[7] << 24);
  o.z = out[8] | (out[9] << 8) | (out[10] << 16) | ((uint32_t)out[11] << 24);
  o.w = out[12] | (out[13] << 8) | (out[14] << 16) | ((uint32_t)out[15] << 24);
  *reinterpret_cast<uint4*>(tdst + kMxCodeBytes + o0) = o;
}

__global__ void pack_mx_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                               int E, int rows, int K, int layout, int RB, int C,
                               uint8_t* __restrict__ dst, int* err, int umma) {
  const int rows_half = rows / 2;  // gate/up: I
  const long long per_tile = 1024 + 64;
  const long long units = (long long)E * RB * C * per_tile;
  const int kb_total = K / 32;
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < units;
       u += (long long)gridDim.x * blockDim.x) {
    const long long tile = u / per_tile;
    const int v = (int)(u % per_tile);
    const int e = (int)(tile / ((long long)RB * C));
    const int rem = (int)(tile % ((long long)RB * C));
    const int rb = rem / C, c = rem % C;
    const uint8_t* ce = codes + (long long)e * rows * (K / 2);
    const uint8_t* se = scales + (long long)e * rows * kb_total;
    uint8_t* tdst = dst + tile * kMxTileBytes;
    if (umma) {
      pack_mx_umma_unit(ce, se, layout, rb, c, rows, rows_half, K, v, tdst, err);
      continue;
    }
    uint8_t out[16];
    if (v < 1024) {
      const int lane = v & 31, bp = (v >> 5) & 3, w = v >> 7;
      const int g = lane >> 2, t = lane & 3;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int b = 2 * bp + (j >> 3), r = j & 7, s = r >> 2, q = r & 3;
        const int row_in_block = 16 * w + frag_row(g, q);
        const int k0 = c * kMxChunkK + 32 * b + frag_k(t, s, q, 0);  // even
        bool valid;
        const int sr = mx_src_row(layout, rb, row_in_block, rows_half, rows, valid);
        out[j] = (valid && k0 < K) ? ce[(long long)sr * (K / 2) + k0 / 2] : 0;
      }
      uint4 o;
      o.x = out[0] | (out[1] << 8) | (out[2] << 16) | ((uint32_t)out[3] << 24);
      o.y = out[4] | (out[5] << 8) | (out[6] << 16) | ((uint32_t)out[7] << 24);
      o.z = out[8] | (out[9] << 8) | (out[10] << 16) | ((uint32_t)out[11] << 24);
      o.w = out[12] | (out[13] << 8) | (out[14] << 16) | ((uint32_t)out[15] << 24);
      *reinterpret_cast<uint4*>(tdst + (w * 4 + bp) * 512 + lane * 16) = o;
    } else {
      const int idx = v - 1024, w = idx >> 3, g = idx & 7;
      int bad = 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int row_in_block = 16 * w + g + ((j >= 8) ? 8 : 0);
        const int blk = c * 8 + (j & 7);
        bool valid;
        const int sr = mx_src_row(layout, rb, row_in_block, rows_half, rows, valid);
        uint8_t sv = 127;
        if (valid && blk < kb_total) {
          sv = se[(long long)sr * kb_total + blk];
          if (sv == 0xFF) bad = 1;
        }
        out[j] = sv;
      }
      if (bad) atomicOr(err, 1 << ERR_NAN_SCALE);
      uint4 o;
      o.x = out[0] | (out[1] << 8) | (out[2] << 16) | ((uint32_t)out[3] << 24);
      o.y = out[4] | (out[5] << 8) | (out[6] << 16) | ((uint32_t)out[7] << 24);
      o.z = out[8] | (out[9] << 8) | (out[10] << 16) | ((uint32_t)out[11] << 24);
      o.w = out[12] | (out[13] << 8) | (out[14] << 16) | ((uint32_t)out[15] << 24);
      *reinterpret_cast<uint4*>(tdst + kMxCodeBytes + (w * 8 + g) * 16) = o;
    }
  }
}

int launch_pack_dense(const void* src, int K, int N, int layout, int RB, int C, int /*rows_valid*/,
                      uint8_t* dst, void* stream, const void* src2, int K2, int C_first, int umma) {
  const long long units = (long long)RB * C * 1024;
  const int threads = 256;
  const int blocks = (int)((units + threads - 1) / threads < 65535 * 8 ? (units + threads - 1) / threads
                                                                         : 65535 * 8);
  pack_dense_kernel<<<blocks, threads, 0, (cudaStream_t)stream>>>(
      (const uint16_t*)src, K, N, layout, RB, C, dst, (const uint16_t*)src2, K2, C_first, umma);
  return (int)cudaGetLastError();
}

int launch_pack_mx(const uint8_t* codes, const uint8_t* scales, int E, int rows, int K, int layout,
                   int RB, int C, uint8_t* dst, int* err, void* stream, int umma) {
  const long long units = (long long)E * RB * C * (1024 + 64);
  const int threads = 256;
  long long nb = (units + threads - 1) / threads;
  if (nb > 65535LL * 16) nb = 65535LL * 16;
  pack_mx_kernel<<<(int)nb, threads, 0, (cudaStream_t)stream>>>(codes, scales, E, rows, K, layout,
                                                                 RB, C, dst, err, umma);
  return (int)cudaGetLastError();
}

}  // namespace moe
