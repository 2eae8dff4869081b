// Host-side launch state that depends on the device: kernel attributes that are set once
// before a kernel's first launch, and the SM count that sizes persistent grids.  Both are
// kept per device and guarded by one mutex, so the first forwards may come from several
// host threads, each on its own stream, and from several devices at once.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <set>
#include <utility>

namespace focr {
namespace launch_state {
constexpr int kMaxDevices = 64;
inline std::mutex& mutex() {
    static std::mutex m;
    return m;
}
inline std::set<std::pair<int, const void*>>& done() {
    static std::set<std::pair<int, const void*>> s;
    return s;
}
inline int* sms() {
    static int a[kMaxDevices] = {};
    return a;
}
}  // namespace launch_state

// SM count of the current device (0 if it cannot be queried).
inline int device_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= launch_state::kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(launch_state::mutex());
    int& s = launch_state::sms()[dev];
    if (s == 0 && cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) s = 0;
    return s;
}

// Runs `setup` (returning cudaError_t) once for the pair (current device, key), under the lock;
// a setup that failed runs again on the next call.  `setup` must not call device_sms().
template <class F>
cudaError_t once_per_device(const void* key, F&& setup) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(launch_state::mutex());
    if (launch_state::done().count({dev, key})) return cudaSuccess;
    e = setup();
    if (e == cudaSuccess) launch_state::done().insert({dev, key});
    return e;
}

}  // namespace focr
