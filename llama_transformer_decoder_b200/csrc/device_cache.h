// Per-device state of the host code, safe to use from several host threads.
//
// Kernel attributes (the dynamic shared-memory limit) belong to one device
// context and device properties (the SM count) to one device: a process that
// drives two GPUs must set the attribute on each of them and may see
// different SM counts. The caches below are keyed by an integer the caller
// chooses (a context id or a device ordinal). This header has no CUDA
// dependency so that its logic can be tested on a machine without a GPU.
#pragma once
#include <cstdint>
#include <map>
#include <mutex>
#include <set>
#include <utility>

namespace llama {

// Runs a set-up step once per (context or device, key). A step that fails (returns
// non-zero) is not remembered, so the next call tries again. The lock is held
// while the step runs: two threads never set up the same pair at once.
class OncePerDevice {
 public:
  template <typename Setup>
  int run(uint64_t dev, const void* key, Setup&& setup) {
    std::lock_guard<std::mutex> lk(mu_);
    const std::pair<uint64_t, const void*> k(dev, key);
    if (done_.count(k)) return 0;
    const int rc = setup();
    if (rc == 0) done_.insert(k);
    return rc;
  }
  bool done(uint64_t dev, const void* key) {
    std::lock_guard<std::mutex> lk(mu_);
    return done_.count(std::pair<uint64_t, const void*>(dev, key)) != 0;
  }

 private:
  std::mutex mu_;
  std::set<std::pair<uint64_t, const void*>> done_;
};

// A value computed once per device (e.g. a device attribute). `query` returns
// the value, or a value <= 0 when it failed; failures are not cached and the
// caller's fallback is returned instead.
template <typename V>
class PerDeviceValue {
 public:
  template <typename Query>
  V get(int dev, Query&& query, V fallback) {
    std::lock_guard<std::mutex> lk(mu_);
    auto it = vals_.find(dev);
    if (it != vals_.end()) return it->second;
    const V v = query();
    if (v <= V(0)) return fallback;
    vals_[dev] = v;
    return v;
  }

 private:
  std::mutex mu_;
  std::map<int, V> vals_;
};

}  // namespace llama
