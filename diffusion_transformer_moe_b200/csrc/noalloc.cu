// nmoe_forward_noalloc: the whole layer with its scratch in a fixed device array.
//
// Some callers cannot allocate device memory at the point where they run the layer:
// code that runs under a memory manager owning every byte of the device (a caching
// allocator or a pre-partitioned arena), real-time paths that must not enter the CUDA
// allocator, or hosts that forbid allocation after start-up. For them this entry point
// keeps every intermediate of the layer (scores, chosen tokens, token lists, H, Y) in
// one file-scope __device__ array of kStaticScratchBytes, reserved on each device that
// loads this code and held until the process exits. It calls no cudaMalloc, cudaFree
// or other allocating routine.
//
// Host code cannot use the array's name as a device address (it is a host-side stand-
// in), so each device's address is looked up once with cudaGetSymbolAddress, with that
// device current, on the first call made on that device.
#include <mutex>

#include "nmoe_internal.cuh"

// NMOE_NOALLOC_SCRATCH_BYTES (128 MiB): enough for T = 8192, d = 2048, E = 64, F = 1024,
// C = 128 with the default (split) intermediates, which need about 100 MiB.
constexpr size_t kStaticScratchBytes = NMOE_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char nmoe_static_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// The device address of the array on the current device (looked up once per device).
nmoe_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return NMOE_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, nmoe_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return NMOE_ERR_CUDA;
    }
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return NMOE_OK;
}

}  // namespace

extern "C" {

nmoe_status nmoe_forward_noalloc(const void* x, const void* W_r, const void* W1,
                                 const void* W3, const void* W2, int64_t T, int64_t d,
                                 int64_t E, int64_t F, int64_t C, void* out,
                                 nmoe_stream_t stream) {
  nmoe_options o;
  nmoe_options_init(&o);
  const size_t need = nmoe_workspace_size(T, d, E, F, C, &o);
  if (need > kStaticScratchBytes) return NMOE_ERR_WORKSPACE;
  void* ws = nullptr;
  nmoe_status st = scratch_address(&ws);
  if (st != NMOE_OK) return st;
  // Nothing in the scratch has to start at zero: every intermediate is written in full
  // before it is read, so the previous call's contents are never observed.
  o.workspace = ws;
  o.workspace_bytes = kStaticScratchBytes;
  return nmoe_forward_ex(x, W_r, W1, W3, W2, T, d, E, F, C, out, stream, &o);
}

}  // extern "C"
