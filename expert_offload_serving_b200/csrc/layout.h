// Expert blob layout, shared by the CUDA kernels (through common.cuh) and the
// host-compiled expert kernel: offsets of every weight, scale and tile inside
// one expert's blob.  Plain inline functions, callable on host and device.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/moe.h"

#if defined(__CUDACC__)
#define MOE_HD __host__ __device__
#else
#define MOE_HD
#endif

namespace moe {

// ---------------------------------------------------------------- blob layout
// One expert = one blob; every region starts on a 256-byte boundary.
//   BF16 : wg [I][d], wu [I][d], wd [d][I] (bf16; row-major, or in the
//          tensor-core tile layout when bf16_blocked(d, I) -- sw128_offset).
//   MXFP4: codes wg [I][d/2], wu [I][d/2], wd [d][I/2] (low nibble = even
//          element), then E8M0 scales sg [I][d/32], su [I][d/32], sd [d][I/32].
//   NVFP4: codes of W_gu [2I][d/2] -- gate and up rows interleaved in blocks
//          of 64 (rows 128b..128b+63 = gate rows 64b.., rows 128b+64.. = up
//          rows 64b..), so one 128-row tensor-core tile holds the gate and up
//          rows of the same 64 intermediate indices -- then W_d [d][I/2];
//          E4M3 scales of W_gu and W_d in tensor-core atoms (sf_atom_offset);
//          then 3 fp32 tensor scales (gate, up, down).  wu/su alias wg/sg.
struct BlobLayout {
  size_t wg, wu, wd, sg, su, sd, ts, bytes;
};

MOE_HD inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

MOE_HD inline BlobLayout blob_layout(int fmt, int d, int I) {
  BlobLayout L{};
  size_t m = static_cast<size_t>(I) * d;   // elements of one matrix
  size_t o = 0;
  if (fmt == MOE_W_BF16) {
    L.wg = o; o = round_up(o + m * 2, 256);
    L.wu = o; o = round_up(o + m * 2, 256);
    L.wd = o; o = round_up(o + m * 2, 256);
    L.sg = L.su = L.sd = L.ts = o;
  } else if (fmt == MOE_W_MXFP4 && d % 256 == 0 && I % 256 == 0) {
    // stage-tiled (mx_tile_code_offset): W_gu tiles, then W_d tiles; the
    // scale regions alias the code regions
    L.wg = L.wu = L.sg = L.su = o; o = round_up(o + m + m / 16, 256);
    L.wd = L.sd = o; o = round_up(o + m / 2 + m / 32, 256);
    L.ts = o;
  } else if (fmt == MOE_W_MXFP4) {
    L.wg = o; o = round_up(o + m / 2, 256);
    L.wu = o; o = round_up(o + m / 2, 256);
    L.wd = o; o = round_up(o + m / 2, 256);
    L.sg = o; o = round_up(o + m / 32, 256);
    L.su = o; o = round_up(o + m / 32, 256);
    L.sd = o; o = round_up(o + m / 32, 256);
    L.ts = o;
  } else {
    L.wg = L.wu = o; o = round_up(o + m, 256);         // W_gu codes
    L.wd = o; o = round_up(o + m / 2, 256);
    L.sg = L.su = o; o = round_up(o + m / 8, 256);     // W_gu scales
    L.sd = o; o = round_up(o + m / 16, 256);
    L.ts = o; o = round_up(o + 3 * sizeof(float), 256);
  }
  L.bytes = o;
  return L;
}

// bf16 blobs whose d and I are multiples of 256 store their matrices in the
// tensor-core tile layout of the decode GEMV: W_gu = the gate and up rows
// interleaved in blocks of 64 (gu_row), occupying the wg and wu regions as one
// [2I][d] matrix, and W_d [d][I]; each as tiles of 128 rows x 64 elements
// (16 KB), ordered [row / 128][k / 64], so a tile's K range is contiguous and
// one pipeline stage is one bulk copy.  Inside a tile row r is a 128-byte line
// whose 16-byte chunk c (8 elements) sits at c ^ (r % 8): the canonical
// 128-byte-swizzled K-major operand layout of tcgen05.mma.
MOE_HD inline bool bf16_blocked(int d, int I) { return d % 256 == 0 && I % 256 == 0; }

// Byte offset of element (r, k) of a tile-layout matrix with K columns.
MOE_HD inline size_t sw128_offset(int r, int k, int K) {
  const size_t tile = static_cast<size_t>(r >> 7) * (K >> 6) + (k >> 6);
  const int rr = r & 127, c = (k >> 3) & 7;
  return tile * 16384 + static_cast<size_t>(rr) * 128 + ((c ^ (rr & 7)) << 4) + (k & 7) * 2;
}

// MXFP4 blobs whose d and I are multiples of 256 are stage-tiled for the
// tensor-core decode GEMV: W_gu (gate and up rows interleaved as in gu_row)
// and W_d are cut into tiles of 128 rows x 256 elements, ordered
// [row / 128][k / 256], each 17408 bytes: the codes (row r = 128 bytes at
// 128 r, element 2i in the low nibble of byte i; the TMA expands and swizzles
// them on the way into shared memory), then the E8M0 scales as two
// scale-factor atoms of the tensor core (sf_atom_offset's layout: atom a holds
// the tile's 32-element blocks 4a..4a+3).  One tile is one pipeline stage and
// one contiguous L2 prefetch.
MOE_HD inline bool mx_tiled(int d, int I) { return d % 256 == 0 && I % 256 == 0; }
constexpr int kMxTileBytes = 128 * 128 + 128 * 8;

// Byte offsets of code byte b (elements 2b, 2b+1) and of the scale of 32-block
// j of row r, in a stage-tiled matrix with K columns.
MOE_HD inline size_t mx_tile_code_offset(int r, int b, int K) {
  const size_t tile = static_cast<size_t>(r >> 7) * (K >> 8) + (b >> 7);
  return tile * kMxTileBytes + static_cast<size_t>(r & 127) * 128 + (b & 127);
}
MOE_HD inline size_t mx_tile_scale_offset(int r, int j, int K) {
  const size_t tile = static_cast<size_t>(r >> 7) * (K >> 8) + (j >> 3);
  const int rr = r & 127, jj = j & 7;
  return tile * kMxTileBytes + 16384 + (jj >> 2) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (jj & 3);
}

// Row of W_gu holding gate row i (up = false) or up row i (up = true).
MOE_HD inline int gu_row(int i, bool up) { return (i >> 6) * 128 + (up ? 64 : 0) + (i & 63); }

// Byte offset of the E4M3 scale of (row r, 16-element block b) of an NVFP4
// matrix with K columns, in the scale-factor atom layout the FP4 tensor-core
// MMA reads: atoms of 128 rows x 4 blocks (512 bytes), atoms ordered
// [row/128][block/4]; inside an atom row r sits at (r%32)*16 + ((r/32)%4)*4
// and block b at b%4.
MOE_HD inline size_t sf_atom_offset(int r, int b, int K) {
  return (static_cast<size_t>(r >> 7) * (K >> 6) + (b >> 2)) * 512 +
         (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

}  // namespace moe
