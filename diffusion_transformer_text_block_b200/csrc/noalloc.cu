// Allocation-free variant of the timestep-modulation pipeline.
//
// The regular path (moss_op_modulation and every forward) keeps the timesteps and the
// conditioning vectors SiLU(c) in workspace that moss_model_create allocated.  This file
// offers the same computation to callers that may not allocate device memory at all: the
// scratch lives in one file-scope __device__ array of fixed size, present on every GPU that
// loads the library for as long as the process runs.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "../../include/moss_dit.h"
#include "internal.h"

namespace moss {
namespace {

struct NoAllocScratch {
  float t[MOSS_NOALLOC_MAX_TIMESTEPS];
  float sc[MOSS_NOALLOC_MAX_TIMESTEPS * MOSS_NOALLOC_MAX_COND_DIM];
};

// 64 KB + 256 B per device.  Host code must not use this name as a device address: its
// address is looked up with cudaGetSymbolAddress below.
static __device__ __align__(256) NoAllocScratch g_noalloc_scratch;

struct TimeArgs {
  float t[MOSS_NOALLOC_MAX_TIMESTEPS];
};

// Timesteps arrive by value in the kernel parameters, so no host-to-device copy is needed.
__global__ void store_timesteps(TimeArgs a, int n) {
  if (static_cast<int>(threadIdx.x) < n) g_noalloc_scratch.t[threadIdx.x] = a.t[threadIdx.x];
}

std::mutex g_mu;
NoAllocScratch* g_scratch_addr[64] = {nullptr};

// Device address of the scratch array on the current device, looked up once per device.
cudaError_t scratch_address(NoAllocScratch** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<NoAllocScratch*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moss

using namespace moss;

extern "C" int moss_modulation_noalloc(const moss_config* cfg, const moss_weights* w, const float* t_host, int n_t,
                                       float* mod_out, void* stream) {
  if (!cfg || !w || !t_host || !mod_out)
    return set_error(MOSS_ERR_INVALID_ARGUMENT, "cfg, w, t_host and mod_out must not be NULL");
  if (cfg->struct_size != sizeof(moss_config) || w->struct_size != sizeof(moss_weights))
    return set_error(MOSS_ERR_ABI_MISMATCH, "struct_size not accepted by this library");
  if (n_t < 1 || n_t > MOSS_NOALLOC_MAX_TIMESTEPS)
    return set_error(MOSS_ERR_INVALID_ARGUMENT,
                     "n_t must be in 1..MOSS_NOALLOC_MAX_TIMESTEPS (64): the fixed scratch holds no more");
  if (cfg->cond_dim < 32 || cfg->cond_dim > MOSS_NOALLOC_MAX_COND_DIM || cfg->cond_dim % 32)
    return set_error(MOSS_ERR_INVALID_ARGUMENT,
                     "cond_dim must be a multiple of 32 up to MOSS_NOALLOC_MAX_COND_DIM (256)");
  if (cfg->layers < 1 || cfg->hidden < 1)
    return set_error(MOSS_ERR_INVALID_ARGUMENT, "layers and hidden must be positive");
  const void* ptrs[] = {w->t_w1, w->t_b1, w->t_w2, w->t_b2, w->mod_w, w->mod_b, w->final_mod_w, w->final_mod_b};
  for (const void* p : ptrs)
    if (!p || !aligned16(p))
      return set_error(MOSS_ERR_INVALID_ARGUMENT, "modulation weight pointers must be non-NULL and 16-byte aligned");
  if (!aligned16(mod_out)) return set_error(MOSS_ERR_INVALID_ARGUMENT, "mod_out must be 16-byte aligned");

  NoAllocScratch* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess)
    return set_error(MOSS_ERR_CUDA, std::string("scratch address lookup: ") + cudaGetErrorString(e));

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = cfg->hidden, L = cfg->layers, C = cfg->cond_dim;
  const int64_t stride = static_cast<int64_t>(L) * 6 * D + 2 * D;
  TimeArgs args{};
  for (int i = 0; i < n_t; ++i) args.t[i] = t_host[i];
  count_launches(4);
  store_timesteps<<<1, MOSS_NOALLOC_MAX_TIMESTEPS, 0, s>>>(args, n_t);
  e = cudaGetLastError();
  // Every element of scratch->sc[0 .. n_t*C) is overwritten by the conditioning kernel before
  // the GEMV reads it, so nothing left from an earlier call is ever read.
  if (e == cudaSuccess)
    e = launch_conditioning(static_cast<const bf16*>(w->t_w1), static_cast<const bf16*>(w->t_b1),
                            static_cast<const bf16*>(w->t_w2), static_cast<const bf16*>(w->t_b2), scratch->t,
                            scratch->sc, n_t, C, s);
  if (e == cudaSuccess)
    e = launch_mod_gemv(static_cast<const bf16*>(w->mod_w), static_cast<const bf16*>(w->mod_b), scratch->sc, mod_out,
                        L * 6 * D, C, n_t, stride, s);
  if (e == cudaSuccess)
    e = launch_mod_gemv(static_cast<const bf16*>(w->final_mod_w), static_cast<const bf16*>(w->final_mod_b),
                        scratch->sc, mod_out + static_cast<int64_t>(L) * 6 * D, 2 * D, C, n_t, stride, s);
  if (e != cudaSuccess) return set_error(MOSS_ERR_CUDA, std::string("modulation: ") + cudaGetErrorString(e));
  return set_error(MOSS_OK, "");
}
