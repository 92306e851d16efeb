// moe_permute_noalloc: moe_permute for callers that cannot allocate device
// memory.
//
// moe_permute needs a small scratch buffer (per-block expert counts and their
// prefix sums) that the caller passes in.  Some callers have no way to get
// one: an inference step running inside an engine that has reserved all of
// HBM up front (KV cache, weights) and forbids allocation while a step runs,
// or a plugin or custom-op interface whose host hands it only its input and
// output tensors.  For them this entry point uses a buffer that lives in the
// library itself: a file-scope __device__ array of fixed size, one per device
// that loads the library, held until the process exits.
//
// Rules of use:
//  - The first call on a device looks up the array's device address with
//    that device current (cudaGetSymbolAddress); make that first call before
//    any stream capture on the device.
//  - All calls on a device share the one array.  Calls whose work overlaps on
//    the GPU (different streams, no ordering between them) race on it and
//    give wrong results; serialise them on one stream.
//  - The array keeps the previous call's contents.  That is harmless here:
//    the counting pass writes every entry before the later passes read it,
//    so nothing needs clearing.
//  - A problem needing more scratch than the array holds is rejected with
//    MOE_ERR_UNSUPPORTED before anything is launched.
//  - The looked-up address is kept for the life of the process.  After a
//    cudaDeviceReset() the module is loaded again and the array may move, so
//    a process that resets a device must not call this entry point on it
//    again (use moe_permute with its own workspace, or a fresh process).
#include <atomic>

#include "common.cuh"

namespace {

// 1 MiB: enough for T*k up to 524288 routed entries at E = 256, or 4.19M at E = 32.
constexpr size_t kScratchBytes = 1u << 20;

static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_addr[kMaxDevices];

// Device address of the scratch array for the current device, looked up once
// per device with that device current.  (In host code the array's name is
// only a host-side stand-in, never a device address.)  Host threads that make
// their first call on a device at the same time may both look it up; they
// find the same address, and the slot is atomic.
int scratch_address(void **scratch)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *scratch = p;
    return MOE_OK;
}

}  // namespace

extern "C" int moe_permute_noalloc(const int32_t *idx, const moe_dims *d, int32_t *counts, int32_t *offsets,
                                   int32_t *pos, int32_t *src_idx, const uint16_t *x, uint8_t *xq, float *xs,
                                   void *stream)
{
    if (!d || d->T < 0 || d->D <= 0 || d->E <= 0 || d->k <= 0) return MOE_ERR_INVALID_ARG;
    if (d->align != 1 && d->align != 128) return MOE_ERR_INVALID_ARG;
    if (d->E > 256 || d->k > 16 || d->k > d->E || d->D % 128) return MOE_ERR_UNSUPPORTED;
    if (!counts || !offsets || !src_idx) return MOE_ERR_INVALID_ARG;
    if (d->T > 0 && (!idx || !pos)) return MOE_ERR_INVALID_ARG;
    auto a16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (x && (!xq || !xs || !a16(x) || !a16(xq) || (reinterpret_cast<uintptr_t>(xs) & 3u))) return MOE_ERR_INVALID_ARG;
    if (moe::permute_ws_bytes(d->T, d->k, d->E) > kScratchBytes) return MOE_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    int st = scratch_address(&scratch);
    if (st) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int64_t r = (int64_t)d->T * d->k + (int64_t)d->E * (d->align - 1);
    const int64_t R_cap = (r + 127) / 128 * 128;
    // Routing entries outside [0, E) are dropped (pos = -1) as in moe_permute,
    // but not reported through moe_get_status().
    st = moe::launch_permute_index(idx, d->T, d->k, d->E, d->align, counts, offsets, pos, src_idx, R_cap, scratch,
                                   nullptr, s);
    if (st || !x) return st;
    st = moe::launch_quant_1x128(x, d->D, d->T, d->D, pos, d->k, xq, d->D, xs, R_cap, s);
    if (st) return st;
    return moe::launch_pad_rows(counts, offsets, d->E, d->D, R_cap, xq, xs, nullptr, s);
}
