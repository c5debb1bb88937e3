// Host state the launchers keep per GPU: kernel attributes that must be set (the
// dynamic shared-memory limit, non-portable cluster sizes) and occupancy answers
// (how many CTA pairs fit) are properties of one device's context, so each device
// gets its own entry, filled the first time a kernel runs there.  One process may
// therefore drive layers on several GPUs, one after another or from several
// threads.
//
// Plain C++ (no CUDA types): the same code is compiled by the host compiler in a
// CPU test that drives it with fake devices.
#pragma once
#include <atomic>
#include <mutex>

namespace ttt {

constexpr int kPerDeviceSlots = 64;

// Set-up that must succeed once per device: `run(dev, f)` calls f() the first
// time device `dev` asks, and again after a failed attempt (f returns non-zero);
// once f has returned 0 for a device it is never called for it again.  Devices
// outside [0, kPerDeviceSlots) are not cached: f runs every time.
class OncePerDevice {
 public:
  template <class F>
  int run(int dev, F&& f) {
    if (dev < 0 || dev >= kPerDeviceSlots) return static_cast<int>(f());
    if (done_[dev].load(std::memory_order_acquire)) return 0;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_[dev].load(std::memory_order_relaxed)) return 0;
    const int r = static_cast<int>(f());
    if (r == 0) done_[dev].store(true, std::memory_order_release);
    return r;
  }

 private:
  std::mutex mu_;
  std::atomic<bool> done_[kPerDeviceSlots] = {};
};

// A value computed once per device: `get(dev, f)` returns f()'s result for that
// device, computing it the first time the device asks.  Devices outside
// [0, kPerDeviceSlots) are not cached.
class IntPerDevice {
 public:
  template <class F>
  int get(int dev, F&& f) {
    if (dev < 0 || dev >= kPerDeviceSlots) return f();
    if (has_[dev].load(std::memory_order_acquire)) return val_[dev];
    std::lock_guard<std::mutex> lock(mu_);
    if (!has_[dev].load(std::memory_order_relaxed)) {
      val_[dev] = f();
      has_[dev].store(true, std::memory_order_release);
    }
    return val_[dev];
  }

 private:
  std::mutex mu_;
  std::atomic<bool> has_[kPerDeviceSlots] = {};
  int val_[kPerDeviceSlots] = {};
};

}  // namespace ttt
