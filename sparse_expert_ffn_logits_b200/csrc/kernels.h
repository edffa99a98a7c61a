// kernels.h - host-side launchers of the layer's kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "tma.cuh"

namespace moe {

struct LaunchShape {
  int nsm;            // SMs of the device
  int grid_gate;      // persistent grid of the gate kernel
  int grid_updown;    // persistent grid of the up/down kernel
  int grid_select;    // cap of the selection grid
  Ring ring_gate;     // copy ring of the bf16 gate kernel
  Ring ring_ud;       // copy ring of the bf16 up/down kernel
  Ring ring_layer;    // copy ring of the fused layer kernel (ns = 0: not available)
  int variant;        // register-fragment ring variant (0: generic token tiles in smem)
  int router_cluster; // CTAs of the single-cluster router (0: only the multi-CTA router)
};

constexpr int kMaxDevices = 64;

// Identity of the calling thread's current CUDA context, unique for the life of the process
// (0 if it cannot be read).  A device reset ends a context; the next one has another identity.
unsigned long long current_context_id();

// Held while kernels are configured (function attributes, per-context discoveries), so that
// handles created and routing set up from several threads do not interleave.
std::mutex& setup_mutex();

// dtype: 0 bf16, 1 fp32.  Each launcher returns the launch's cudaError_t.
cudaError_t launch_router(const FwdParams& p, int dtype, cudaStream_t st);
int router_hsplit(int E, int B, int H);
// pdl: launch with programmatic stream serialization (off while stage timing events are set)
cudaError_t launch_gate(const FwdParams& p, int dtype, const LaunchShape& ls, cudaStream_t st,
                        bool pdl);
cudaError_t launch_select(const FwdParams& p, const LaunchShape& ls, cudaStream_t st, bool pdl);
cudaError_t launch_updown(const FwdParams& p, int dtype, const LaunchShape& ls, cudaStream_t st,
                          bool pdl);
// dense masked fallback (dense.cu): stage 0 = gather + gate GEMM, stage 1 = up + down GEMMs
cudaError_t launch_dense(const FwdParams& p, const LaunchShape& ls, int stage, cudaStream_t st,
                         bool pdl);
cudaError_t configure_dense(int budget);
// fused layer kernel (layer.cu): gate, selection and up/down in one persistent launch
bool layer_available(const LaunchShape& ls);
cudaError_t launch_layer(const FwdParams& p, const LaunchShape& ls, cudaStream_t st, bool pdl);
cudaError_t configure_layer(int H, int imax, int n_slot_max, int smem_budget, LaunchShape* ls);
cudaError_t launch_finalize(const FwdParams& p, int dtype, const LaunchShape& ls, cudaStream_t st,
                            bool pdl);

// Set-up (called once per handle, under setup_mutex): shared-memory limits and persistent grid
// sizes.
cudaError_t configure_kernels(int dtype, int imax, int n_slot_max, int max_B, int H, LaunchShape* ls);
cudaError_t configure_router(int budget, int* cluster_out);
size_t router_smem_bytes(int E, int B);
size_t select_smem_bytes(int imax);

// Packing and debug export.
cudaError_t launch_pack_down(const void* w_down, void* packed_updown, int n, int I, int H,
                             int elt, cudaStream_t st);
cudaError_t launch_force_timeout(const FwdParams& p, cudaStream_t st);
cudaError_t launch_cast_output(const float* sum, void* out, size_t n, int dtype, int nsm,
                               cudaStream_t st);
cudaError_t launch_roster_bias(const int* counts, const int* pinned, int B, int E, int m,
                               float delta, float* bias, cudaStream_t st);
cudaError_t launch_debug_gather(const FwdParams& p, int n_tokens, int* cnt, int* lists,
                                float* act, cudaStream_t st);

// cudaLaunchKernelEx with programmatic stream serialization (the kernel may start while its
// predecessor in the stream runs and calls griddepcontrol.wait before reading its results).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Lets a kernel use all the dynamic shared memory the device allows next to its static shared
// memory.  The attribute is per kernel and per device, so it is always set to this maximum:
// a handle with smaller sizes must never lower the limit under another live handle.
template <typename... KArgs>
cudaError_t allow_max_smem(void (*kernel)(KArgs...), int optin_budget) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin_budget - (int)fa.sharedSizeBytes);
}

}  // namespace moe
