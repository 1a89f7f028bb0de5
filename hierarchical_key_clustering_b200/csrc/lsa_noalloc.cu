// lsa_index_decode_static: the decode indexer for callers that cannot
// allocate device memory.
//
// Who needs it: an engine that reserves all device memory for its KV cache at
// start-up and gives plugins no allocator; a host program that only holds
// device pointers handed to it; a decode loop that must never stall, where a
// cudaMalloc or cudaFree could synchronise the device.  Such callers cannot
// provide the scratch workspace that lsa_index_decode asks for.
//
// This entry point takes its scratch from one fixed array in device memory,
// g_index_scratch below (LSA_STATIC_SCRATCH_BYTES).  Every GPU that loads the
// library holds that array until the process exits.  The call itself
// allocates nothing: it finds the array's device address, checks the request
// fits, and hands the address to lsa_index_decode as its workspace, so the
// kernels and results are exactly those of lsa_index_decode.
//
// In host code, the name g_index_scratch stands for a host-side shadow, not a
// device address: passing it to a kernel would fault, or on a system where the
// GPU can reach host memory, silently use the wrong memory.  The device
// address comes from cudaGetSymbolAddress, done once per device (with that
// device current) on the first call made on it, and kept.
//
// When the array comes into being: under CUDA's default lazy module loading
// a module's device memory (this array, and the code of the kernels the call
// launches) is set up the first time the module is used on a device, not when
// the library is loaded.  So the first call on each device -- even one with
// nq = 0, which does the address look-up and launches nothing -- may allocate
// and synchronise.  Callers should make one call with the sizes they will use
// before they reserve the rest of device memory and before any stream
// capture (or run with CUDA_MODULE_LOADING=EAGER); after that, calls allocate
// nothing.  The kept address assumes the device is never reset
// (cudaDeviceReset) while the library is in use; a reset also ends every
// buffer the caller passes in.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "lsa.h"

namespace lsa {
int report_error(int code, const char *msg);  // sets lsa_last_error_string (lsa_api.cu)
int check_index_params(const lsa_params *p);  // the argument checks of lsa_index_decode (lsa_api.cu)
}

namespace {

static __device__ __align__(256) unsigned char g_index_scratch[LSA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_index_scratch on the current device (set up on the
// first call per device).  Returns 0, a cudaError_t, or -1 for a device
// ordinal this file keeps no slot for.
int scratch_address(void **out, int *dev_out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    *dev_out = dev;
    if (dev < 0 || dev >= kMaxDevices) return -1;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_index_scratch);
        if (e != cudaSuccess) return (int)e;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return 0;
}

}  // namespace

extern "C" int lsa_index_decode_static(const float *qidx, const int64_t *pos, int64_t nq, const lsa_cache *cache,
                                       const lsa_tree *tree, int32_t *lists, int32_t *lens, int32_t Lmax,
                                       const lsa_params *p, void *stream)
{
    // the parameter checks come first, so bad parameters get LSA_ERR_ARG as
    // they do from lsa_index_decode, never a size computed from them
    const int pc = lsa::check_index_params(p);
    if (pc != LSA_OK) return pc;
    if (!cache) return lsa_index_decode(qidx, pos, nq, cache, tree, lists, lens, Lmax, p, nullptr, 0, stream);
    const int64_t need = lsa_index_workspace_bytes(nq, cache->n_blocks, p);
    if (need > (int64_t)LSA_STATIC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "lsa_index_decode_static: %lld queries over %lld blocks need %lld bytes of scratch; the static "
                 "scratch holds %lld (use lsa_index_decode with a workspace)",
                 (long long)nq, (long long)cache->n_blocks, (long long)need, (long long)LSA_STATIC_SCRATCH_BYTES);
        return lsa::report_error(LSA_ERR_WORKSPACE, msg);
    }
    void *ws = nullptr;
    int dev = -1;
    int rc = scratch_address(&ws, &dev);
    if (rc != 0) {
        char msg[256];
        if (rc == -1)
            snprintf(msg, sizeof(msg),
                     "lsa_index_decode_static: device ordinal %d is above the %d devices the static scratch "
                     "keeps addresses for",
                     dev, kMaxDevices - 1);
        else
            snprintf(msg, sizeof(msg),
                     "lsa_index_decode_static: cudaGetSymbolAddress of the static scratch failed on device %d: %s",
                     dev, cudaGetErrorString((cudaError_t)rc));
        return lsa::report_error(LSA_ERR_CUDA, msg);
    }
    return lsa_index_decode(qidx, pos, nq, cache, tree, lists, lens, Lmax, p, ws, (int64_t)LSA_STATIC_SCRATCH_BYTES,
                            stream);
}
