// Paged adapter optimizer on the host CPU.
//
// «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나», § "메모리 회계: 세 겹의 최적화"
// (Paged Optimizer): the adapters' Adam states m and v live in CPU pinned
// memory and the optimizer update runs on the CPU in parallel with the GPU's
// backward, on its own CUDA stream, so the transfers hide behind compute.
//
// qlora_adamw_host is the update itself: AdamW over n parameters held in
// host memory, split across a fixed pool of worker threads owned by the
// library (created on first use, joined at process exit).
//
// qlora_adamw_paged chains the whole page-out step on one stream, fully
// asynchronously: copy the gradient device -> pinned host, run the update as
// a host function of that stream (the CUDA runtime calls it once the copy
// has landed; it calls no CUDA API), and copy the refreshed bf16 adapter
// pinned host -> device. Issued on a second stream after the backward's
// gradients are ready, it overlaps whatever the first stream does next.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <condition_variable>
#include <cstdint>
#include <cstring>
#include <functional>
#include <mutex>
#include <thread>
#include <vector>

#include "../../include/qlora.h"

namespace qlora {
namespace {

// Fixed pool: run(fn, parts) calls fn(0..parts-1) across the workers and the
// calling thread and returns when all parts are done.
class Pool {
 public:
  static Pool& get() {
    static Pool p;
    return p;
  }
  int size() const { return static_cast<int>(workers_.size()) + 1; }

  void run(const std::function<void(int)>& fn, int parts) {
    std::lock_guard<std::mutex> serial(run_mu_);   // one job at a time
    {
      std::lock_guard<std::mutex> lk(mu_);
      fn_ = &fn;
      parts_ = parts;
      next_ = 0;
      done_ = 0;
      ++gen_;
    }
    cv_.notify_all();
    work();
    std::unique_lock<std::mutex> lk(mu_);
    done_cv_.wait(lk, [&] { return done_ == parts_; });
    fn_ = nullptr;
  }

 private:
  Pool() {
    unsigned hc = std::thread::hardware_concurrency();
    int n = static_cast<int>(std::min<unsigned>(hc == 0 ? 4u : hc, 32u)) - 1;
    for (int i = 0; i < n; ++i) workers_.emplace_back([this] { loop(); });
  }
  ~Pool() {
    {
      std::lock_guard<std::mutex> lk(mu_);
      stop_ = true;
    }
    cv_.notify_all();
    for (auto& t : workers_) t.join();
  }
  void work() {
    while (true) {
      int i;
      const std::function<void(int)>* f;
      {
        std::lock_guard<std::mutex> lk(mu_);
        if (fn_ == nullptr || next_ >= parts_) return;
        i = next_++;
        f = fn_;
      }
      (*f)(i);
      std::lock_guard<std::mutex> lk(mu_);
      if (++done_ == parts_) done_cv_.notify_all();
    }
  }
  void loop() {
    uint64_t seen = 0;
    while (true) {
      {
        std::unique_lock<std::mutex> lk(mu_);
        cv_.wait(lk, [&] { return stop_ || (gen_ != seen && fn_ != nullptr && next_ < parts_); });
        if (stop_) return;
        seen = gen_;
      }
      work();
    }
  }
  std::vector<std::thread> workers_;
  std::mutex mu_, run_mu_;
  std::condition_variable cv_, done_cv_;
  const std::function<void(int)>* fn_ = nullptr;
  int parts_ = 0, next_ = 0, done_ = 0;
  uint64_t gen_ = 0;
  bool stop_ = false;
};

inline uint16_t bf16_bits_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return static_cast<uint16_t>((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

struct HostStep {
  float *master, *m, *v;
  const float* grad;
  uint16_t* param;
  int64_t n;
  float beta1, beta2, eps, decay, step_size, inv_sqrt_bc2;
};

void run_step(const HostStep& h) {
  const int parts = std::max(1, std::min<int>(Pool::get().size() * 4, static_cast<int>((h.n + 4095) / 4096)));
  const std::function<void(int)> fn = [&](int part) {
    const int64_t i0 = h.n * part / parts, i1 = h.n * (part + 1) / parts;
    for (int64_t i = i0; i < i1; ++i) {
      const float g = h.grad[i];
      const float m = std::fma(h.beta1, h.m[i], (1.0f - h.beta1) * g);
      const float v = std::fma(h.beta2, h.v[i], (1.0f - h.beta2) * g * g);
      const float denom = std::sqrt(v) * h.inv_sqrt_bc2 + h.eps;
      const float p = h.master[i] * h.decay - h.step_size * (m / denom);
      h.m[i] = m;
      h.v[i] = v;
      h.master[i] = p;
      if (h.param != nullptr) h.param[i] = bf16_bits_rne(p);
    }
  };
  Pool::get().run(fn, parts);
}

bool make_step(HostStep* h, float* master, void* param, const float* grad, float* m, float* v, int64_t n,
               const qlora_adamw_t* hp) {
  if (hp == nullptr || n < 0 || master == nullptr || grad == nullptr || m == nullptr || v == nullptr) return false;
  if (hp->step < 1 || !(hp->lr >= 0.0f) || !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) ||
      !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) || !(hp->eps > 0.0f) || !std::isfinite(hp->weight_decay))
    return false;
  const double bc1 = 1.0 - std::pow(static_cast<double>(hp->beta1), hp->step);
  const double bc2 = 1.0 - std::pow(static_cast<double>(hp->beta2), hp->step);
  *h = HostStep{master, m, v, grad, static_cast<uint16_t*>(param), n, hp->beta1, hp->beta2, hp->eps,
                static_cast<float>(1.0 - static_cast<double>(hp->lr) * hp->weight_decay),
                static_cast<float>(hp->lr / bc1), static_cast<float>(1.0 / std::sqrt(bc2))};
  return true;
}

void CUDART_CB host_step_cb(void* arg) {
  HostStep* h = static_cast<HostStep*>(arg);
  run_step(*h);
  delete h;
}

}  // namespace
}  // namespace qlora

extern "C" {

qlora_status_t qlora_adamw_host(float* master, void* param_bf16, const float* grad, float* m, float* v, int64_t n,
                                const qlora_adamw_t* hp) {
  qlora::HostStep h;
  if (!qlora::make_step(&h, master, param_bf16, grad, m, v, n, hp)) return QLORA_ERR_INVALID_ARG;
  if (n > 0) qlora::run_step(h);
  return QLORA_OK;
}

qlora_status_t qlora_adamw_paged(const float* grad_dev, void* param_dev_bf16, float* master_host, float* m_host,
                                 float* v_host, float* grad_host, void* param_host_bf16, int64_t n,
                                 const qlora_adamw_t* hp, void* stream) {
  if (grad_dev == nullptr || grad_host == nullptr) return QLORA_ERR_INVALID_ARG;
  if ((param_dev_bf16 == nullptr) != (param_host_bf16 == nullptr)) return QLORA_ERR_INVALID_ARG;
  auto* h = new qlora::HostStep;
  if (!qlora::make_step(h, master_host, param_host_bf16, grad_host, m_host, v_host, n, hp)) {
    delete h;
    return QLORA_ERR_INVALID_ARG;
  }
  if (n == 0) {
    delete h;
    return QLORA_OK;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(grad_host, grad_dev, static_cast<size_t>(n) * sizeof(float), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaLaunchHostFunc(st, qlora::host_step_cb, h) != cudaSuccess) {
    delete h;
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  if (param_dev_bf16 != nullptr &&
      cudaMemcpyAsync(param_dev_bf16, param_host_bf16, static_cast<size_t>(n) * 2, cudaMemcpyHostToDevice, st) !=
          cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

}  // extern "C"
