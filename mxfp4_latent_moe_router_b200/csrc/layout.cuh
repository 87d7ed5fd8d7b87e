// layout.cuh -- packed weight tiles and activation records of the B200 path.
//
// Every weight matrix is cut into row blocks of 128 output rows (8 warp tiles
// of 16 rows) and, along K, into chunks; one (row block, chunk) tile is one
// contiguous run of bytes that a single bulk copy moves into shared memory.
// Inside a tile the elements sit in the order in which the lanes of an
// m16n8k16 MMA hold them, so each lane fetches its A fragments with 16-byte
// shared-memory loads and no shuffles.
//
// K permutation.  Within every 32-wide block of K, lane (g = lane/4, t =
// lane%4) covers the 8 physical columns 8t..8t+7: k16 step 0 takes 8t+{0,1}
// (fragment k 2t,2t+1) and 8t+{2,3} (fragment k 2t+8,2t+9), step 1 takes
// 8t+{4,5} and 8t+{6,7}.  The same map is applied to the activations, which
// therefore stay in natural row-major order: lane (g,t) reads 16 bytes of
// token g at columns 32*blk + 8t .. +7.  Each MMA still sums over one 32-wide
// block only, so MX block scales apply after every pair of k16 steps.
#pragma once
#include <cstdint>

namespace moe {

constexpr int kRowsPerBlock = 128;  // rows of one packed row block
constexpr int kWarpRows = 16;       // rows of one warp tile
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + one producer warp

// bf16 tiles: 128 rows x 64 K = 16 KB.  Order: [warp 8][blk 2][step 2][lane 32][16 B]
// with the 16 bytes = 4 A registers (a01 a23 a45 a67) of that k16 step.
constexpr int kDenseChunkK = 64;
constexpr int kDenseTileBytes = kRowsPerBlock * kDenseChunkK * 2;

// MXFP4 tiles: 128 rows x 256 K.  Codes [warp 8][blk pair 4][lane 32][16 B]:
// bytes 0..7 belong to the even block of the pair, 8..15 to the odd one, and
// inside a block byte r (0..7) is A register r%4 of k16 step r/4 as an e2m1
// pair (low nibble = lower k).  Scales follow: [warp 8][g 8][16 B] with bytes
// 0..7 = row g, blocks 0..7 and bytes 8..15 = row g+8, blocks 0..7.
constexpr int kMxChunkK = 256;
constexpr int kMxCodeBytes = kRowsPerBlock * kMxChunkK / 2;  // 16384
constexpr int kMxScaleBytes = kRowsPerBlock * kMxChunkK / 32;  // 1024
constexpr int kMxTileBytes = kMxCodeBytes + kMxScaleBytes;    // 17408

// Activation record for the MXFP4 kernels ("f16 MX"): per (row, 256-wide chunk)
// 256 f16 values scaled by a power of two per 32-block, then the 8 float
// scales that undo it.  544 bytes, 16-byte multiple.
constexpr int kActRecBytes = kMxChunkK * 2 + 8 * 4;

// Tensor-core (tcgen05, kind::mxf4) layouts of the MXFP4 expert kernels,
// selected per plan.  A weight tile keeps its 17408 bytes, reordered for the
// block-scaled MMA's K-major "core matrices" (8 rows x 16 bytes, see
// umma.cuh): the codes as 1024 slots of 16 bytes, slot (kb * 16 + rg) * 8 + r
// holding row rg * 8 + r, K elements 32 kb .. 32 kb + 31 of the chunk (element
// 2t in the low nibble of byte t), so that row groups lie 128 bytes apart and
// K blocks 2048; then the e8m0 scales as two 512-byte units (K blocks 0-3,
// 4-7), byte (m % 32) * 16 + (m / 32) * 4 + kb % 4.
//
// An activation record (per row, 256-wide chunk) holds the value as a sum of
// kUTerms e2m1 terms, each with its own e8m0 scale per 32-block:
//   value = sum_t e2m1(q_t) * 2^(s_t - 127),
// term t's codes packed as 8 K blocks of 16 bytes (128 bytes), then the
// terms' 8 scale bytes each.  Term 1 takes the block maximum to at most 4
// times its scale, each later term a scale 2^-3 of the previous one, and
// each carries what the earlier terms left: the residual after 4 terms is at
// most 2^-11 of the block maximum.
constexpr int kUTerms = 4;
constexpr int kUTermBytes = kMxChunkK / 2;                      // 128
constexpr int kActRecBytesU = kUTerms * kUTermBytes + kUTerms * 8;  // 544

// A tensor-core ring stage: [header 128][A: packed codes 16 KB][A scales
// 1 KB][B: kUTerms * 8 NT token-term rows of 128 bytes][B scales 1 KB]
constexpr int kUHdrBytes = 128;
constexpr int kUAOff = kUHdrBytes;
constexpr int kUSfaOff = kUAOff + kMxCodeBytes;
constexpr int kUBOff = kUSfaOff + kMxScaleBytes;
__host__ __device__ constexpr int umma_rows(int nt) { return kUTerms * 8 * nt; }
__host__ __device__ constexpr int umma_stage_bytes(int nt) {
  return ((kUBOff + umma_rows(nt) * kUTermBytes + 1024) + 127) / 128 * 128;
}

// fragment map: lane (g,t), k16 step s, register q (0..3), half e (0..1) ->
// (row within the 16-row warp tile, physical k within the 32-block)
__host__ __device__ constexpr int frag_row(int g, int q) { return (q & 1) ? g + 8 : g; }
__host__ __device__ constexpr int frag_k(int t, int s, int q, int e) {
  return 8 * t + 4 * s + ((q & 2) ? 2 : 0) + e;
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Pieces per row block (split-K factor) for `mats` row blocks of C chunks
// each, dealt dynamically to `ctas` CTAs.  A dynamic schedule ends within one
// piece of the average load, and CTAs arrive skewed, so the estimate is
//   total work / ctas + one piece,
// a piece costing its chunks plus, when split, split_cost: the price of a
// split-K piece end (partial sums out, a ticket, sometimes the finalising
// sums) in chunk-stage units.
__host__ __device__ inline int best_ppr(int mats, int C, int ctas, int split_cost) {
  if (mats <= 0 || ctas <= 0 || C <= 1) return 1;
  int best = 1;
  long long best_t = -1;
  for (int ppr = 1; ppr <= C; ++ppr) {
    const long long piece = ceil_div(C, ppr) + (ppr > 1 ? split_cost : 0);
    const long long t = ((long long)mats * ppr * piece + ctas - 1) / ctas + piece;
    if (best_t < 0 || t < best_t) {
      best_t = t;
      best = ppr;
    }
  }
  return best;
}

}  // namespace moe
