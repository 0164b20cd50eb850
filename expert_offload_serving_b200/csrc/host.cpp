// Host-only parts of libmoe: error strings, shape checks, device attributes,
// and moe_pack_expert (canonical tensors -> device-final expert blob).
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace moe {

static thread_local char g_err[512] = "";

moe_status fail(moe_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

void clear_error() { g_err[0] = '\0'; }

namespace {
std::atomic<uint64_t> g_wait_ns{2000000000ull};
std::atomic<int> g_stall{0};
}

uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }
int test_stall() { return g_stall.load(std::memory_order_relaxed); }

moe_status check_shape(moe_shape s) {
  MOE_REQUIRE(s.E >= 1 && s.E <= 1024, "E=%d outside [1, 1024]", s.E);
  MOE_REQUIRE(s.d >= 1 && s.I >= 1 && s.d <= 16384 && s.I <= 16384,
              "d=%d, I=%d outside [1, 16384]", s.d, s.I);
  if (s.fmt == MOE_W_BF16) {
    MOE_REQUIRE(s.d % 8 == 0 && s.I % 8 == 0, "BF16 needs d, I multiples of 8 (d=%d, I=%d)", s.d, s.I);
  } else if (s.fmt == MOE_W_MXFP4) {
    MOE_REQUIRE(s.d % 32 == 0 && s.I % 32 == 0, "MXFP4 needs d, I multiples of 32 (d=%d, I=%d)", s.d, s.I);
  } else if (s.fmt == MOE_W_NVFP4) {
    MOE_REQUIRE(s.d % 128 == 0 && s.I % 128 == 0, "NVFP4 needs d, I multiples of 128 (d=%d, I=%d)", s.d, s.I);
  } else {
    return fail(MOE_ERR_INVALID_ARG, "unknown weight format %d", s.fmt);
  }
  return MOE_OK;
}

moe_status current_device(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device id %d", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    DeviceInfo d{};
    d.id = dev;
    MOE_CUDA_TRY(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev));
    MOE_CUDA_TRY(cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev));
    MOE_CUDA_TRY(cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev));
    int optin = 0;
    MOE_CUDA_TRY(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    d.smem_optin = static_cast<size_t>(optin);
    cache[dev] = d;
    have[dev] = true;
  }
  *out = cache[dev];
  if (out->cc_major != 10)
    return fail(MOE_ERR_UNSUPPORTED, "libmoe is built for sm_100a; device %d is sm_%d%d",
                dev, out->cc_major, out->cc_minor);
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" int moe_abi_version(void) { return 1; }

extern "C" int moe_set_test_stall(int on) { return g_stall.exchange(on ? 1 : 0); }

extern "C" uint64_t moe_set_wait_limit_ns(uint64_t ns) {
  const uint64_t prev = g_wait_ns.load();
  g_wait_ns.store(ns == 0 ? 2000000000ull : ns);
  return prev;
}

extern "C" const char* moe_last_error(void) { return g_err; }

extern "C" size_t moe_expert_blob_bytes(moe_shape s) {
  if (check_shape(s) != MOE_OK) return 0;
  return blob_layout(s.fmt, s.d, s.I).bytes;
}

extern "C" moe_status moe_pack_expert(moe_shape s, const void* wg, const void* wu, const void* wd,
                                      const uint8_t* sg, const uint8_t* su, const uint8_t* sd,
                                      const float* tensor_scales, void* blob_out) {
  clear_error();
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(wg && wu && wd && blob_out, "null weight or output pointer");
  const BlobLayout L = blob_layout(s.fmt, s.d, s.I);
  uint8_t* b = static_cast<uint8_t*>(blob_out);
  std::memset(b, 0, L.bytes);
  const size_t m = static_cast<size_t>(s.I) * s.d;
  if (s.fmt == MOE_W_BF16) {
    if (!bf16_blocked(s.d, s.I)) {
      std::memcpy(b + L.wg, wg, m * 2);
      std::memcpy(b + L.wu, wu, m * 2);
      std::memcpy(b + L.wd, wd, m * 2);
      return MOE_OK;
    }
    // tile layout: gate/up rows interleaved into W_gu, 16-byte chunks to their
    // swizzled places
    const uint8_t* g8 = static_cast<const uint8_t*>(wg);
    const uint8_t* u8 = static_cast<const uint8_t*>(wu);
    const uint8_t* d8 = static_cast<const uint8_t*>(wd);
    for (int i = 0; i < s.I; ++i)
      for (int k = 0; k < s.d; k += 8) {
        const size_t src = (static_cast<size_t>(i) * s.d + k) * 2;
        std::memcpy(b + L.wg + sw128_offset(gu_row(i, false), k, s.d), g8 + src, 16);
        std::memcpy(b + L.wg + sw128_offset(gu_row(i, true), k, s.d), u8 + src, 16);
      }
    for (int r = 0; r < s.d; ++r)
      for (int k = 0; k < s.I; k += 8)
        std::memcpy(b + L.wd + sw128_offset(r, k, s.I), d8 + (static_cast<size_t>(r) * s.I + k) * 2, 16);
    return MOE_OK;
  }
  MOE_REQUIRE(sg && su && sd, "null scale pointer for an FP4 format");
  if (s.fmt == MOE_W_MXFP4 && mx_tiled(s.d, s.I)) {
    // stage tiles: 16-byte code chunks to their rows, scale bytes into the
    // tiles' scale-factor atoms
    const uint8_t* cg = static_cast<const uint8_t*>(wg);
    const uint8_t* cu = static_cast<const uint8_t*>(wu);
    const uint8_t* cd = static_cast<const uint8_t*>(wd);
    for (int i = 0; i < s.I; ++i) {
      const int rg = gu_row(i, false), ru = gu_row(i, true);
      for (int bb = 0; bb < s.d / 2; bb += 16) {
        std::memcpy(b + L.wg + mx_tile_code_offset(rg, bb, s.d), cg + static_cast<size_t>(i) * (s.d / 2) + bb, 16);
        std::memcpy(b + L.wg + mx_tile_code_offset(ru, bb, s.d), cu + static_cast<size_t>(i) * (s.d / 2) + bb, 16);
      }
      for (int j = 0; j < s.d / 32; ++j) {
        b[L.wg + mx_tile_scale_offset(rg, j, s.d)] = sg[static_cast<size_t>(i) * (s.d / 32) + j];
        b[L.wg + mx_tile_scale_offset(ru, j, s.d)] = su[static_cast<size_t>(i) * (s.d / 32) + j];
      }
    }
    for (int r = 0; r < s.d; ++r) {
      for (int bb = 0; bb < s.I / 2; bb += 16)
        std::memcpy(b + L.wd + mx_tile_code_offset(r, bb, s.I), cd + static_cast<size_t>(r) * (s.I / 2) + bb, 16);
      for (int j = 0; j < s.I / 32; ++j)
        b[L.wd + mx_tile_scale_offset(r, j, s.I)] = sd[static_cast<size_t>(r) * (s.I / 32) + j];
    }
    return MOE_OK;
  }
  if (s.fmt == MOE_W_MXFP4) {
    std::memcpy(b + L.wg, wg, m / 2);
    std::memcpy(b + L.wu, wu, m / 2);
    std::memcpy(b + L.wd, wd, m / 2);
    std::memcpy(b + L.sg, sg, m / 32);
    std::memcpy(b + L.su, su, m / 32);
    std::memcpy(b + L.sd, sd, m / 32);
    return MOE_OK;
  }
  MOE_REQUIRE(tensor_scales != nullptr, "NVFP4 needs 3 tensor scales");
  // W_gu: gate and up rows interleaved in blocks of 64; scale bytes move from
  // row-major [R][K/16] into the MMA atom layout
  const size_t gate_row_bytes = static_cast<size_t>(s.d) / 2;
  const int nbd = s.d / 16;
  for (int i = 0; i < s.I; ++i) {
    const int rg = gu_row(i, false), ru = gu_row(i, true);
    std::memcpy(b + L.wg + rg * gate_row_bytes, static_cast<const uint8_t*>(wg) + i * gate_row_bytes,
                gate_row_bytes);
    std::memcpy(b + L.wg + ru * gate_row_bytes, static_cast<const uint8_t*>(wu) + i * gate_row_bytes,
                gate_row_bytes);
    for (int blk = 0; blk < nbd; ++blk) {
      b[L.sg + sf_atom_offset(rg, blk, s.d)] = sg[static_cast<size_t>(i) * nbd + blk];
      b[L.sg + sf_atom_offset(ru, blk, s.d)] = su[static_cast<size_t>(i) * nbd + blk];
    }
  }
  std::memcpy(b + L.wd, wd, m / 2);
  const int nbi = s.I / 16;
  for (int r = 0; r < s.d; ++r)
    for (int blk = 0; blk < nbi; ++blk)
      b[L.sd + sf_atom_offset(r, blk, s.I)] = sd[static_cast<size_t>(r) * nbi + blk];
  std::memcpy(b + L.ts, tensor_scales, 3 * sizeof(float));
  return MOE_OK;
}
