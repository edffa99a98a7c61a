// synth_host.cpp - host fill of the seeded input generator (definition in synth.h).
// Compiled with -ffp-contract=off so that the host and device fills agree bit for bit.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <thread>
#include <vector>

#include "synth.h"

namespace {

void fill_range(void* dst, int64_t begin, int64_t end, uint64_t key, uint64_t offset, double stdv,
                int dtype) {
  for (int64_t i = begin; i < end; ++i) {
    double z = synth_mul(synth_normal(key, offset + (uint64_t)i), stdv);
    float f = synth_to_f32(z);
    if (dtype == SYNTH_BF16) {
      static_cast<uint16_t*>(dst)[i] = synth_f32_to_bf16(f);
    } else {
      static_cast<float*>(dst)[i] = f;
    }
  }
}

}  // namespace

extern "C" {

// Fills dst[0..n) with elements offset..offset+n-1 of tensor (seed, tensor_id), scaled by stdv
// and rounded to dtype (SYNTH_BF16: uint16 bit patterns, SYNTH_F32: binary32).
// nthreads <= 0 uses every hardware thread.  Returns 0, or -1 on a bad argument.
int synth_fill_host(void* dst, int64_t n, uint64_t seed, uint64_t tensor_id, uint64_t offset,
                    double stdv, int dtype, int nthreads) {
  if (n < 0 || (n > 0 && dst == nullptr) || (dtype != SYNTH_BF16 && dtype != SYNTH_F32)) return -1;
  if (n == 0) return 0;
  uint64_t key = synth_key(seed, tensor_id);
  int hw = (int)std::thread::hardware_concurrency();
  int nt = nthreads > 0 ? nthreads : (hw > 0 ? hw : 1);
  int64_t per = std::max<int64_t>(1 << 16, (n + nt - 1) / nt);
  std::vector<std::thread> pool;
  for (int64_t b = 0; b < n; b += per) {
    int64_t e = std::min<int64_t>(n, b + per);
    pool.emplace_back(fill_range, dst, b, e, key, offset, stdv, dtype);
  }
  for (auto& t : pool) t.join();
  return 0;
}

// Number of hardware threads the host fill uses by default.
int synth_host_threads(void) {
  int hw = (int)std::thread::hardware_concurrency();
  return hw > 0 ? hw : 1;
}

}  // extern "C"
