// focr_moe_layer_forward_noalloc: the layer forward without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at the point where they run the layer:
// a plug-in or callback hosted by an application that owns the whole device memory
// budget and hands out no allocator, or latency-critical code that must not call
// cudaMalloc because it can block and synchronise the device.  Those callers still
// own the input and output buffers, but cannot provide the router/dispatch scratch
// the regular forward takes.  This variant uses a fixed scratch array that lives in
// the library's own device image instead: every GPU that loads the library holds it
// (FOCR_NOALLOC_SCRATCH_BYTES) until the process exits.
//
// The array is named below; in host code that name is only a stand-in, not a device
// address, so the host looks the address up with cudaGetSymbolAddress once per device
// (with that device current) and hands the looked-up pointer to the kernels.
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace focr {
focr_status report_error(focr_status s, const char* msg);
}

using namespace focr;

namespace {

constexpr WsLayout kNoallocLayout = ws_layout(FOCR_NOALLOC_T_MAX, IS);
static_assert(kNoallocLayout.total == FOCR_NOALLOC_SCRATCH_BYTES, "header constant out of date");
// control words, k-split partial sums and their counters: zero before the first forward and
// left zero by every forward that completes
constexpr size_t kZeroBytes = kNoallocLayout.gpart;

static __device__ __align__(256) unsigned char g_noalloc_scratch[FOCR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

focr_status noalloc_fail(focr_status s, const char* fmt, int a, int b) {
    char buf[256];
    snprintf(buf, sizeof(buf), fmt, a, b);
    return report_error(s, buf);
}

// Device address of the scratch array on the current device; the first call per device
// looks it up and zero-fills it (synchronously).
focr_status scratch_for_current_device(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return report_error(FOCR_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(FOCR_ERR_UNSUPPORTED, "device %d >= %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) return report_error(FOCR_ERR_CUDA, cudaGetErrorString(e));
        e = cudaMemset(p, 0, FOCR_NOALLOC_SCRATCH_BYTES);
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return report_error(FOCR_ERR_CUDA, cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return FOCR_OK;
}

}  // namespace

extern "C" focr_status focr_moe_layer_forward_noalloc(const focr_moe_layer* layer, const float* hidden, int32_t T,
                                                      float* out, const focr_moe_route_debug* dbg, void* stream) {
    if (T < 1 || T > FOCR_NOALLOC_T_MAX)
        return noalloc_fail(FOCR_ERR_INVALID_ARG, "T=%d outside [1, %d], the fixed scratch limit", T,
                            FOCR_NOALLOC_T_MAX);
    void* scratch = nullptr;
    focr_status s = scratch_for_current_device(&scratch);
    if (s != FOCR_OK) return s;
    // Nothing is cleared per call: the array's zero prefix is zero after the first-use fill
    // and every forward that completes leaves it zero.  A forward whose bounded device wait
    // ran out may leave it dirty; focr_moe_check_noalloc reports that and restores it.
    return focr_moe_layer_forward(layer, hidden, T, out, scratch, FOCR_NOALLOC_SCRATCH_BYTES, dbg, stream);
}

extern "C" focr_status focr_moe_check_noalloc(void* stream) {
    void* scratch = nullptr;
    focr_status s = scratch_for_current_device(&scratch);
    if (s != FOCR_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    int32_t* err = reinterpret_cast<int32_t*>((char*)scratch + kNoallocLayout.ctrl) + CTRL_ERROR;
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, err, sizeof(v), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return report_error(FOCR_ERR_CUDA, cudaGetErrorString(e));
    if (v == 0) return FOCR_OK;
    if (v == DEVERR_RANGE) {   // the forward completed; only the word is cleared
        const int32_t zero = 0;
        e = cudaMemcpyAsync(err, &zero, sizeof(zero), cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return report_error(FOCR_ERR_CUDA, cudaGetErrorString(e));
        return report_error(FOCR_ERR_RANGE, "activations beyond the f16 operand range (|v| > 65504) met by a forward");
    }
    // a wait ran out: the forward that set the word may have left counters and partial sums
    // behind, so the whole zero prefix (the error word included) is cleared
    e = cudaMemsetAsync(scratch, 0, kZeroBytes, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return report_error(FOCR_ERR_CUDA, cudaGetErrorString(e));
    char buf[96];
    snprintf(buf, sizeof(buf), "device wait ran out (code %d); the scratch array was cleared", v);
    return report_error(FOCR_ERR_TIMEOUT, buf);
}
