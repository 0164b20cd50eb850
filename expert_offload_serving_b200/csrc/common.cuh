// Shared definitions of libmoe: error reporting, argument checks, the expert
// blob layout, and small device helpers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

// ---------------------------------------------------------------- errors
moe_status fail(moe_status st, const char* fmt, ...);
void clear_error();

#define MOE_REQUIRE(cond, ...)                                   \
  do {                                                           \
    if (!(cond)) return ::moe::fail(MOE_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define MOE_CUDA_TRY(call)                                                        \
  do {                                                                            \
    cudaError_t e_ = (call);                                                      \
    if (e_ != cudaSuccess)                                                        \
      return ::moe::fail(MOE_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

#define MOE_LAUNCH_CHECK(what)                                                    \
  do {                                                                            \
    cudaError_t e_ = cudaGetLastError();                                          \
    if (e_ != cudaSuccess)                                                        \
      return ::moe::fail(MOE_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e_)); \
  } while (0)

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Device attributes of the current device (cached per device id).
struct DeviceInfo { int id, sm_count, cc_major, cc_minor; size_t smem_optin; };
moe_status current_device(DeviceInfo* out);

// ---------------------------------------------------------------- blob layout
// One expert = one blob; every region starts on a 256-byte boundary.
//   BF16 : wg [I][d], wu [I][d], wd [d][I] (bf16; row-major, or blocked when
//          bf16_blocked(d, I) -- see blocked_offset).
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

__host__ __device__ inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline BlobLayout blob_layout(int fmt, int d, int I) {
  BlobLayout L{};
  size_t m = static_cast<size_t>(I) * d;   // elements of one matrix
  size_t o = 0;
  if (fmt == MOE_W_BF16) {
    L.wg = o; o = round_up(o + m * 2, 256);
    L.wu = o; o = round_up(o + m * 2, 256);
    L.wd = o; o = round_up(o + m * 2, 256);
    L.sg = L.su = L.sd = L.ts = o;
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

// bf16 blobs whose d and I are multiples of 256 store each matrix in blocks
// for the decode MMA path: block (rb, ks) = rows [RB*rb, RB*rb + RB) x
// elements [kBlockK*ks, kBlockK*ks + kBlockK), RB = 16 for W_g and W_u, 32 for
// W_d; the blocks of a matrix are ordered [rb][ks], each block holds its rows
// as lines of 2*kBlockK bytes, and inside a line the 16-byte chunk c (8 elements) sits at position
// c ^ (row % 8) -- so one stage of the decode pipeline is one contiguous copy
// and ldmatrix reads of 8 rows hit 8 different bank groups.  Inside every
// group of 32 elements along K the elements are stored in the order
// kpos32: the MMA k-steps 2j and 2j+1 then see, in the B-fragment slots of
// lane group t, the 8 contiguous activations 32j + 8t .. 32j + 8t + 7, which
// the lane fetches with one 16-byte load.
__host__ __device__ inline bool bf16_blocked(int d, int I) { return d % 256 == 0 && I % 256 == 0; }
constexpr int kBlockK = 128;   // elements per line of a block

// Stored position of element k (0..31) of a 32-element group: MMA k-step
// (k >> 2) & 1, fragment register (k >> 1) & 1, lane group k >> 3, half k & 1.
__host__ __device__ inline int kpos32(int k) {
  return ((k >> 2) & 1) * 16 + ((k >> 1) & 1) * 8 + (k >> 3) * 2 + (k & 1);
}

// Byte offset, inside a blocked matrix with K columns, of element (r, k).
__host__ __device__ inline size_t blocked_offset(int r, int k, int K, int RB) {
  const int p = (k & ~31) | kpos32(k & 31);
  const size_t block = static_cast<size_t>(r / RB) * (K / kBlockK) + p / kBlockK;
  const int rr = r % RB, c = (p % kBlockK) >> 3;
  return (block * RB + rr) * (2 * kBlockK) + ((c ^ (rr & 7)) << 4) + (p & 7) * 2;
}

// Row of W_gu holding gate row i (up = false) or up row i (up = true).
__host__ __device__ inline int gu_row(int i, bool up) { return (i >> 6) * 128 + (up ? 64 : 0) + (i & 63); }

// Byte offset of the E4M3 scale of (row r, 16-element block b) of an NVFP4
// matrix with K columns, in the scale-factor atom layout the FP4 tensor-core
// MMA reads: atoms of 128 rows x 4 blocks (512 bytes), atoms ordered
// [row/128][block/4]; inside an atom row r sits at (r%32)*16 + ((r/32)%4)*4
// and block b at b%4.
__host__ __device__ inline size_t sf_atom_offset(int r, int b, int K) {
  return (static_cast<size_t>(r >> 7) * (K >> 6) + (b >> 2)) * 512 +
         (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

moe_status check_shape(moe_shape s);

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

constexpr unsigned kFull = 0xffffffffu;

}  // namespace moe
