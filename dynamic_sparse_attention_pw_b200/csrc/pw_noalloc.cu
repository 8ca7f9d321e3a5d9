// pw_noalloc.cu -- pw_group_noalloc: the grouping call for callers that cannot allocate
// device memory themselves.
//
// pw_group needs a scratch workspace (per-query set sizes, per-group union sizes and union
// bitsets).  Some callers cannot provide one: code that runs where cudaMalloc is not allowed
// (it may synchronise the device, or the host application owns the whole memory budget and
// hands a plug-in only its input and output buffers).  For them this file keeps the scratch
// in a fixed, file-scope device array and passes it to the ordinary pw_group.
//
// The array is allocated by the CUDA runtime when the library's module is loaded on a
// device, so every GPU that loads the library holds it until the process exits.
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/pw.h"

namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(PW_NOALLOC_SCRATCH_BYTES);

// The scratch itself.  In host code this name is only a stand-in for the device object: its
// device address must be fetched with cudaGetSymbolAddress (below), never taken directly.
static __device__ __align__(256) unsigned char g_group_scratch[kNoAllocScratchBytes];

// Device address of g_group_scratch on the current device.  It is looked up on every call:
// the address belongs to the module instance the runtime holds for the device, and a device
// reset replaces that instance, so a cached address could outlive it.  The first lookup on a
// device also loads the module there (with lazy loading), which is why the first call on a
// device should come before any stream capture.
cudaError_t scratch_on_current_device(void **out)
{
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_group_scratch);
    if (e != cudaSuccess)
        return e;
    *out = p;
    return cudaSuccess;
}

} // namespace

extern "C" pw_status pw_group_noalloc(const int32_t *sel_pages, const int32_t *cu_seqlens,
                                      const int32_t *cu_seqlens_host, int B, int Hkv, int kmax,
                                      int W, int g, const pw_groups *groups, int32_t *dev_status,
                                      void *stream)
{
    size_t need = 0;
    const pw_status st =
        pw_groups_size(cu_seqlens_host, B, Hkv, kmax, W, g, nullptr, nullptr, nullptr, &need);
    if (st != PW_OK)
        return st;
    if (need > kNoAllocScratchBytes)
        return PW_ERR_CAPACITY;
    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess)
        return PW_ERR_CUDA;
    // Every byte pw_group reads from its workspace is written earlier in the same call, so
    // the scratch needs no clearing between calls.
    return pw_group(sel_pages, cu_seqlens, cu_seqlens_host, B, Hkv, kmax, W, g, groups, scratch,
                    kNoAllocScratchBytes, dev_status, stream);
}
