// FFN service of Attention-FFN Disaggregation on one host.
//
// The FFN side of an A/F split serves each layer in a loop: take the activations the attention
// side sent, run the layer, send the output back (vLLM AFD Plugin page, section 系統架構,
// "2. FFN Service").  Here the two sides meet in a mailbox of host buffers: the attention side
// posts a micro-batch into a slot and later waits for the slot's output; the serving loop takes
// slots in post order, copies the input to the device, runs afd_ffn_forward and copies the
// output back; a second thread completes each slot as soon as its output has landed.  With two
// or more slots in flight the attention of one micro-batch overlaps the FFN of another (A/F 分离
// page, section 深入推导, 微流水), and the host-to-device copy of one, the layer of another and
// the device-to-host copy of a third run on three streams.
//
// Host code only; every step of the layer is afd_ffn_forward's kernels.  All waits are bounded.
#include "afd_ffn.h"

#include <cuda_runtime.h>
#include <time.h>

#include <atomic>
#include <chrono>
#include <condition_variable>
#include <cstdlib>
#include <cstring>
#include <memory>
#include <mutex>
#include <new>
#include <thread>

namespace {

enum : int { kFree = 0, kPosted = 1, kTaken = 2, kDone = 3, kFailed = 4 };

constexpr int32_t kMaxSlots = 1024;
constexpr int64_t kMaxTimeoutUs = 1000000000000LL;   // ~11.6 days: keeps the deadline in range
constexpr int64_t kPollUs = 100000;                    // serving loop: longest wait between stop checks
constexpr int64_t kSpinNs = 20000;                     // spin this long before sleeping on the mailbox

int64_t now_ns() {
  timespec ts;
  clock_gettime(CLOCK_MONOTONIC, &ts);
  return static_cast<int64_t>(ts.tv_sec) * 1000000000LL + ts.tv_nsec;
}

inline void cpu_relax() {
#if defined(__x86_64__) || defined(__i386__)
  __builtin_ia32_pause();
#endif
}

// Wait until `ready` holds or timeout_us has passed.  A hand-off that comes within kSpinNs is
// caught by spinning; after that the thread sleeps on the mailbox's condition variable, which
// every state change notifies, so an idle side holds no core.
template <class F>
bool wait_until(std::mutex& mu, std::condition_variable& cv, F ready, int64_t timeout_us) {
  if (ready()) return true;
  if (timeout_us < 0) timeout_us = 0;
  if (timeout_us > kMaxTimeoutUs) timeout_us = kMaxTimeoutUs;
  const int64_t t0 = now_ns();
  const int64_t deadline = t0 + timeout_us * 1000;
  const int64_t spin_end = t0 + kSpinNs < deadline ? t0 + kSpinNs : deadline;
  for (int n = 0;; ++n) {
    if (ready()) return true;
    const int64_t t = now_ns();
    if (t >= spin_end) break;
    if (n < 64) cpu_relax(); else std::this_thread::yield();
  }
  std::unique_lock<std::mutex> lk(mu);
  const auto until = std::chrono::steady_clock::now() + std::chrono::nanoseconds(deadline - now_ns());
  return cv.wait_until(lk, until, ready);
}

struct Slot {
  std::atomic<int> state{kFree};
  std::atomic<int32_t> T{0};
  std::atomic<int32_t> status{AFD_OK};
  std::atomic<int64_t> t_post{0}, t_take{0}, t_done{0};
  void* in = nullptr;
  void* out = nullptr;
};

}  // namespace

struct afd_ffn_mailbox {
  int32_t n_slots = 0, T_max = 0, H = 0;
  bool pinned = false;
  size_t buf_bytes = 0;                            // one buffer, T_max * H bf16, 64-byte padded
  void* block = nullptr;                           // all 2 * n_slots buffers
  std::unique_ptr<Slot[]> slots;
  std::unique_ptr<std::atomic<int32_t>[]> ring;    // posted slots in post order
  std::atomic<uint64_t> head{0}, tail{0};          // ring[head % n] is the oldest posted slot
  std::mutex post_mu, take_mu;
  std::mutex mu;                                   // sleeping waiters: state changes notify cv
  std::condition_variable cv;
  std::atomic<bool> served{false};                 // a service consumes this mailbox
};

namespace {

bool bad_slot(const afd_ffn_mailbox* mb, int32_t slot) { return !mb || slot < 0 || slot >= mb->n_slots; }

// Wake every sleeping waiter.  Taking the lock once after the change means a waiter that
// tested the old state under the lock is already asleep, so it cannot miss this notification.
void notify(afd_ffn_mailbox* mb) {
  { std::lock_guard<std::mutex> g(mb->mu); }
  mb->cv.notify_all();
}

}  // namespace

extern "C" {

int afd_ffn_mailbox_create(int32_t n_slots, int32_t T_max, int32_t H, int32_t flags, afd_ffn_mailbox** out) {
  if (!out) return AFD_ERR_INVALID_ARG;
  *out = nullptr;
  if (n_slots < 1 || n_slots > kMaxSlots || T_max < 1 || H < 8 || H % 8 || (flags & ~AFD_MAILBOX_PINNED))
    return AFD_ERR_INVALID_ARG;
  const size_t raw = static_cast<size_t>(T_max) * static_cast<size_t>(H) * 2;
  const size_t buf = (raw + 63) & ~static_cast<size_t>(63);
  const size_t total = buf * 2 * static_cast<size_t>(n_slots);
  afd_ffn_mailbox* mb = new (std::nothrow) afd_ffn_mailbox;
  if (!mb) return AFD_ERR_INVALID_ARG;
  mb->slots.reset(new (std::nothrow) Slot[n_slots]);
  mb->ring.reset(new (std::nothrow) std::atomic<int32_t>[n_slots]);
  if (!mb->slots || !mb->ring) {
    delete mb;
    return AFD_ERR_INVALID_ARG;
  }
  mb->n_slots = n_slots;
  mb->T_max = T_max;
  mb->H = H;
  mb->buf_bytes = buf;
  mb->pinned = (flags & AFD_MAILBOX_PINNED) != 0;
  if (mb->pinned) {
    if (cudaHostAlloc(&mb->block, total, cudaHostAllocPortable) != cudaSuccess) {
      mb->block = nullptr;
      delete mb;
      return AFD_ERR_CUDA;
    }
  } else {
    mb->block = std::aligned_alloc(64, total);
    if (!mb->block) {
      delete mb;
      return AFD_ERR_INVALID_ARG;
    }
  }
  std::memset(mb->block, 0, total);
  char* base = static_cast<char*>(mb->block);
  for (int32_t i = 0; i < n_slots; ++i) {
    mb->slots[i].in = base + (2 * static_cast<size_t>(i)) * buf;
    mb->slots[i].out = base + (2 * static_cast<size_t>(i) + 1) * buf;
    mb->ring[i].store(0, std::memory_order_relaxed);
  }
  *out = mb;
  return AFD_OK;
}

void afd_ffn_mailbox_destroy(afd_ffn_mailbox* mb) {
  if (!mb) return;
  if (mb->block) {
    if (mb->pinned) cudaFreeHost(mb->block); else std::free(mb->block);
  }
  delete mb;
}

void* afd_ffn_mailbox_input(afd_ffn_mailbox* mb, int32_t slot) {
  return bad_slot(mb, slot) ? nullptr : mb->slots[slot].in;
}

void* afd_ffn_mailbox_output(afd_ffn_mailbox* mb, int32_t slot) {
  return bad_slot(mb, slot) ? nullptr : mb->slots[slot].out;
}

int afd_ffn_mailbox_post(afd_ffn_mailbox* mb, int32_t slot, int32_t T) {
  if (bad_slot(mb, slot) || T < 0 || T > mb->T_max) return AFD_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(mb->post_mu);
  Slot& s = mb->slots[slot];
  const int st = s.state.load(std::memory_order_acquire);
  if (st == kPosted || st == kTaken) return AFD_ERR_INVALID_ARG;
  s.T.store(T, std::memory_order_relaxed);
  s.status.store(AFD_OK, std::memory_order_relaxed);
  s.t_take.store(0, std::memory_order_relaxed);
  s.t_done.store(0, std::memory_order_relaxed);
  s.t_post.store(now_ns(), std::memory_order_relaxed);
  s.state.store(kPosted, std::memory_order_release);
  // at most n_slots slots are posted and not yet taken, so the ring never overruns its head
  const uint64_t t = mb->tail.load(std::memory_order_relaxed);
  mb->ring[t % static_cast<uint64_t>(mb->n_slots)].store(slot, std::memory_order_relaxed);
  mb->tail.store(t + 1, std::memory_order_release);
  notify(mb);
  return AFD_OK;
}

int afd_ffn_mailbox_wait(afd_ffn_mailbox* mb, int32_t slot, int64_t timeout_us) {
  if (bad_slot(mb, slot)) return AFD_ERR_INVALID_ARG;
  Slot& s = mb->slots[slot];
  int st = s.state.load(std::memory_order_acquire);
  if (st == kFree) return AFD_ERR_INVALID_ARG;
  const bool ended = wait_until(mb->mu, mb->cv, [&] {
    st = s.state.load(std::memory_order_acquire);
    return st == kDone || st == kFailed;
  }, timeout_us);
  if (!ended) return AFD_ERR_TIMEOUT;
  return st == kDone ? AFD_OK : s.status.load(std::memory_order_relaxed);
}

}  // extern "C"

namespace {

// take, returning AFD_ERR_TIMEOUT early once *cancel is set (the serving loop's stop flag)
int take_slot(afd_ffn_mailbox* mb, int32_t* slot, int32_t* T, int64_t timeout_us,
              const std::atomic<bool>* cancel) {
  if (!mb || !slot || !T) return AFD_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(mb->take_mu);
  const uint64_t h = mb->head.load(std::memory_order_relaxed);
  const bool posted = wait_until(mb->mu, mb->cv, [&] {
    return mb->tail.load(std::memory_order_acquire) > h || (cancel && cancel->load(std::memory_order_acquire));
  }, timeout_us);
  if (!posted || mb->tail.load(std::memory_order_acquire) <= h) return AFD_ERR_TIMEOUT;
  const int32_t sl = mb->ring[h % static_cast<uint64_t>(mb->n_slots)].load(std::memory_order_relaxed);
  mb->head.store(h + 1, std::memory_order_release);
  Slot& s = mb->slots[sl];
  s.t_take.store(now_ns(), std::memory_order_relaxed);
  s.state.store(kTaken, std::memory_order_release);
  *slot = sl;
  *T = s.T.load(std::memory_order_relaxed);
  return AFD_OK;
}

}  // namespace

extern "C" {

int afd_ffn_mailbox_take(afd_ffn_mailbox* mb, int32_t* slot, int32_t* T, int64_t timeout_us) {
  return take_slot(mb, slot, T, timeout_us, nullptr);
}

int afd_ffn_mailbox_complete(afd_ffn_mailbox* mb, int32_t slot, int32_t status) {
  if (bad_slot(mb, slot) || status > 0) return AFD_ERR_INVALID_ARG;
  Slot& s = mb->slots[slot];
  if (s.state.load(std::memory_order_acquire) != kTaken) return AFD_ERR_INVALID_ARG;
  s.status.store(status, std::memory_order_relaxed);
  s.t_done.store(now_ns(), std::memory_order_relaxed);
  s.state.store(status == AFD_OK ? kDone : kFailed, std::memory_order_release);
  notify(mb);
  return AFD_OK;
}

int afd_ffn_mailbox_times(afd_ffn_mailbox* mb, int32_t slot, int64_t* times_ns) {
  if (bad_slot(mb, slot) || !times_ns) return AFD_ERR_INVALID_ARG;
  const Slot& s = mb->slots[slot];
  times_ns[0] = s.t_post.load(std::memory_order_relaxed);
  times_ns[1] = s.t_take.load(std::memory_order_relaxed);
  times_ns[2] = s.t_done.load(std::memory_order_relaxed);
  return AFD_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------ serving loop
namespace {

constexpr int64_t kLandNs = 60LL * 1000000000LL;   // give up on a micro-batch's output after 60 s

}  // namespace

struct afd_ffn_service {
  afd_ffn_handle* h = nullptr;
  afd_ffn_mailbox* mb = nullptr;
  int device = 0;
  cudaStream_t stream = nullptr;                      // the caller's stream: the layer
  cudaStream_t copy_in = nullptr, copy_out = nullptr; // owned
  std::unique_ptr<void*[]> din, dout;                 // per slot, device [T_max][H] bf16
  std::unique_ptr<cudaEvent_t[]> ev_h2d, ev_in, ev_start, ev_fwd, ev_out;   // timing events per slot
  cudaEvent_t ev_origin = nullptr;                     // recorded once when the loop is set up
  std::thread thread, completer;
  std::atomic<bool> stop{false};
  std::atomic<int64_t> served{0};
  std::atomic<int32_t> status{AFD_OK};         // first failure of the loop or the completer
  std::atomic<int32_t> last_cuda_error{0};
  int32_t device_status = AFD_OK;
  // slots whose D2H is enqueued, oldest first; the completer finishes them in this order
  std::mutex fl_mu;
  std::condition_variable fl_cv;
  std::unique_ptr<int32_t[]> in_flight;        // ring of n_slots entries
  uint64_t fl_head = 0, fl_tail = 0;           // under fl_mu
  bool loop_done = false;                      // under fl_mu: no more slots will be enqueued
};

namespace {

int note_cuda(afd_ffn_service* v, cudaError_t e) {
  v->last_cuda_error.store(static_cast<int32_t>(e));
  return AFD_ERR_CUDA;
}

void fail(afd_ffn_service* v, int32_t st) {
  int32_t ok = AFD_OK;
  v->status.compare_exchange_strong(ok, st);
}

#define SVC_CUDA(v, call)                              \
  do {                                                 \
    cudaError_t e_ = (call);                           \
    if (e_ != cudaSuccess) return note_cuda((v), e_);  \
  } while (0)

// Enqueue one micro-batch: H2D on copy_in, the layer on the caller's stream, D2H on copy_out,
// and hand the slot to the completer, which completes it once the D2H has landed.  A slot is
// re-posted only after it completed, so its buffers are free again; the event waits say so to
// the device as well.
int serve_one(afd_ffn_service* v, int32_t slot, int32_t T) {
  Slot& s = v->mb->slots[slot];
  const size_t bytes = static_cast<size_t>(T) * static_cast<size_t>(v->mb->H) * 2;
  SVC_CUDA(v, cudaStreamWaitEvent(v->copy_in, v->ev_fwd[slot], 0));
  SVC_CUDA(v, cudaEventRecord(v->ev_h2d[slot], v->copy_in));
  if (bytes) SVC_CUDA(v, cudaMemcpyAsync(v->din[slot], s.in, bytes, cudaMemcpyHostToDevice, v->copy_in));
  SVC_CUDA(v, cudaEventRecord(v->ev_in[slot], v->copy_in));
  SVC_CUDA(v, cudaStreamWaitEvent(v->stream, v->ev_in[slot], 0));
  SVC_CUDA(v, cudaStreamWaitEvent(v->stream, v->ev_out[slot], 0));
  SVC_CUDA(v, cudaEventRecord(v->ev_start[slot], v->stream));
  const int st = afd_ffn_forward(v->h, v->din[slot], T, v->dout[slot], v->stream);
  if (st != AFD_OK) {
    if (st == AFD_ERR_CUDA) v->last_cuda_error.store(afd_ffn_last_cuda_error(v->h));
    return st;
  }
  SVC_CUDA(v, cudaEventRecord(v->ev_fwd[slot], v->stream));
  SVC_CUDA(v, cudaStreamWaitEvent(v->copy_out, v->ev_fwd[slot], 0));
  if (bytes) SVC_CUDA(v, cudaMemcpyAsync(s.out, v->dout[slot], bytes, cudaMemcpyDeviceToHost, v->copy_out));
  SVC_CUDA(v, cudaEventRecord(v->ev_out[slot], v->copy_out));
  {
    std::lock_guard<std::mutex> g(v->fl_mu);
    v->in_flight[v->fl_tail++ % static_cast<uint64_t>(v->mb->n_slots)] = slot;
  }
  v->fl_cv.notify_one();
  return AFD_OK;
}

// The completer: for each enqueued slot in order, poll the event after its D2H and complete the
// slot as soon as the output is in host memory.  Polling costs this thread's core while
// micro-batches are in flight and gives the attention side the output within microseconds; it
// sleeps when nothing is in flight.
void complete_loop(afd_ffn_service* v) {
  cudaSetDevice(v->device);
  for (;;) {
    int32_t slot;
    {
      std::unique_lock<std::mutex> lk(v->fl_mu);
      v->fl_cv.wait(lk, [&] { return v->fl_head < v->fl_tail || v->loop_done; });
      if (v->fl_head == v->fl_tail) return;          // the loop has ended and nothing is left
      slot = v->in_flight[v->fl_head++ % static_cast<uint64_t>(v->mb->n_slots)];
    }
    cudaError_t e = cudaErrorNotReady;
    const int64_t give_up = now_ns() + kLandNs;
    for (int n = 0;; ++n) {
      e = cudaEventQuery(v->ev_out[slot]);
      if (e != cudaErrorNotReady || now_ns() > give_up) break;
      if (n < 256) cpu_relax(); else std::this_thread::yield();
    }
    if (e == cudaSuccess) {
      if (afd_ffn_mailbox_complete(v->mb, slot, AFD_OK) == AFD_OK) v->served.fetch_add(1);
    } else {
      const int32_t st = e == cudaErrorNotReady ? AFD_ERR_TIMEOUT : note_cuda(v, e);
      fail(v, st);
      afd_ffn_mailbox_complete(v->mb, slot, st);
    }
  }
}

void drain(afd_ffn_service* v) {
  cudaStreamSynchronize(v->copy_in);
  cudaStreamSynchronize(v->stream);
  cudaStreamSynchronize(v->copy_out);
}

void end_completer(afd_ffn_service* v) {
  {
    std::lock_guard<std::mutex> g(v->fl_mu);
    v->loop_done = true;
  }
  v->fl_cv.notify_one();
  if (v->completer.joinable()) v->completer.join();
}

void serve_loop(afd_ffn_service* v) {
  if (cudaSetDevice(v->device) != cudaSuccess) fail(v, AFD_ERR_NO_DEVICE);
  while (!v->stop.load(std::memory_order_acquire)) {
    int32_t slot = 0, T = 0;
    if (take_slot(v->mb, &slot, &T, kPollUs, &v->stop) != AFD_OK) continue;
    int st = v->status.load();
    if (st == AFD_OK && (st = serve_one(v, slot, T)) != AFD_OK) {
      fail(v, st);
      drain(v);     // nothing of this slot may still be reading or writing its buffers
    }
    if (st != AFD_OK) afd_ffn_mailbox_complete(v->mb, slot, st);
  }
  end_completer(v);   // every enqueued slot is completed before this returns
  drain(v);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) fail(v, note_cuda(v, e));
  // posted but never taken
  int32_t slot = 0, T = 0;
  while (afd_ffn_mailbox_take(v->mb, &slot, &T, 0) == AFD_OK) afd_ffn_mailbox_complete(v->mb, slot, AFD_ERR_STOPPED);
  // taken but never completed (cannot happen after the completer drained; kept as a guard)
  const int32_t end_st = v->status.load() != AFD_OK ? v->status.load() : AFD_ERR_CUDA;
  for (int32_t i = 0; i < v->mb->n_slots; ++i) afd_ffn_mailbox_complete(v->mb, i, end_st);   // no-op unless taken
  v->device_status = afd_ffn_get_error(v->h);
}

void release(afd_ffn_service* v) {
  const int32_t n = v->mb ? v->mb->n_slots : 0;
  for (int32_t i = 0; i < n; ++i) {
    if (v->din && v->din[i]) cudaFree(v->din[i]);
    if (v->dout && v->dout[i]) cudaFree(v->dout[i]);
    std::unique_ptr<cudaEvent_t[]>* const evsets[] = {&v->ev_h2d, &v->ev_in, &v->ev_start, &v->ev_fwd, &v->ev_out};
    for (auto* evs : evsets)
      if (*evs && (*evs)[i]) cudaEventDestroy((*evs)[i]);
  }
  if (v->ev_origin) cudaEventDestroy(v->ev_origin);
  if (v->copy_in) cudaStreamDestroy(v->copy_in);
  if (v->copy_out) cudaStreamDestroy(v->copy_out);
  if (v->mb) v->mb->served.store(false, std::memory_order_release);
  delete v;
}

int setup(afd_ffn_service* v) {
  const int32_t n = v->mb->n_slots;
  const size_t bytes = static_cast<size_t>(v->mb->T_max) * static_cast<size_t>(v->mb->H) * 2;
  v->din.reset(new (std::nothrow) void*[n]());
  v->dout.reset(new (std::nothrow) void*[n]());
  std::unique_ptr<cudaEvent_t[]>* const evsets[] = {&v->ev_h2d, &v->ev_in, &v->ev_start, &v->ev_fwd, &v->ev_out};
  for (auto* evs : evsets) evs->reset(new (std::nothrow) cudaEvent_t[n]());
  v->in_flight.reset(new (std::nothrow) int32_t[n]());
  if (!v->din || !v->dout || !v->ev_h2d || !v->ev_in || !v->ev_start || !v->ev_fwd || !v->ev_out || !v->in_flight)
    return AFD_ERR_INVALID_ARG;
  SVC_CUDA(v, cudaStreamCreateWithFlags(&v->copy_in, cudaStreamNonBlocking));
  SVC_CUDA(v, cudaStreamCreateWithFlags(&v->copy_out, cudaStreamNonBlocking));
  SVC_CUDA(v, cudaEventCreate(&v->ev_origin));
  SVC_CUDA(v, cudaEventRecord(v->ev_origin, v->copy_in));
  for (int32_t i = 0; i < n; ++i) {
    SVC_CUDA(v, cudaMalloc(&v->din[i], bytes));
    SVC_CUDA(v, cudaMalloc(&v->dout[i], bytes));
    for (auto* evs : evsets) SVC_CUDA(v, cudaEventCreate(&(*evs)[i]));
  }
  return AFD_OK;
}

}  // namespace

extern "C" {

int afd_ffn_service_start(afd_ffn_handle* h, afd_ffn_mailbox* mb, void* stream, afd_ffn_service** out) {
  if (!out) return AFD_ERR_INVALID_ARG;
  *out = nullptr;
  if (!h || !mb) return AFD_ERR_INVALID_ARG;
  afd_ffn_cfg cfg;
  int32_t dev = -1;
  if (afd_ffn_get_info(h, &cfg, &dev) != AFD_OK) return AFD_ERR_INVALID_ARG;
  if (cfg.H != mb->H || cfg.T_max < mb->T_max) return AFD_ERR_INVALID_ARG;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return AFD_ERR_NO_DEVICE;
  if (cur != dev) return AFD_ERR_INVALID_ARG;
  bool idle = false;
  if (!mb->served.compare_exchange_strong(idle, true)) return AFD_ERR_INVALID_ARG;   // one service per mailbox
  afd_ffn_service* v = new (std::nothrow) afd_ffn_service;
  if (!v) {
    mb->served.store(false);
    return AFD_ERR_INVALID_ARG;
  }
  v->h = h;
  v->mb = mb;
  v->device = dev;
  v->stream = static_cast<cudaStream_t>(stream);
  int st = setup(v);
  if (st != AFD_OK) {
    release(v);
    return st;
  }
  try {
    v->completer = std::thread(complete_loop, v);
  } catch (...) {
    release(v);
    return AFD_ERR_UNSUPPORTED;     // no host thread could be started
  }
  try {
    v->thread = std::thread(serve_loop, v);
  } catch (...) {
    end_completer(v);
    release(v);
    return AFD_ERR_UNSUPPORTED;
  }
  *out = v;
  return AFD_OK;
}

int afd_ffn_service_stop(afd_ffn_service* v, afd_ffn_service_stats* stats) {
  if (!v) return AFD_ERR_INVALID_ARG;
  v->stop.store(true, std::memory_order_release);
  notify(v->mb);
  if (v->thread.joinable()) v->thread.join();
  const int32_t status = v->status.load();
  if (stats) {
    stats->served = v->served.load();
    stats->status = status;
    stats->device_status = v->device_status;
    stats->last_cuda_error = v->last_cuda_error.load();
    stats->reserved = 0;
  }
  release(v);
  return status;
}

}  // extern "C"

extern "C" int afd_ffn_service_slot_timeline(afd_ffn_service* v, int32_t slot, float* ms) {
  if (!v || !ms || slot < 0 || slot >= v->mb->n_slots) return AFD_ERR_INVALID_ARG;
  if (v->mb->slots[slot].state.load(std::memory_order_acquire) != kDone) return AFD_ERR_INVALID_ARG;
  const cudaEvent_t t0 = v->ev_h2d[slot];
  const cudaEvent_t ends[4] = {v->ev_in[slot], v->ev_start[slot], v->ev_fwd[slot], v->ev_out[slot]};
  cudaError_t e = cudaEventElapsedTime(&ms[0], v->ev_origin, t0);
  for (int i = 0; i < 4 && e == cudaSuccess; ++i) e = cudaEventElapsedTime(&ms[1 + i], t0, ends[i]);
  return e == cudaSuccess ? AFD_OK : AFD_ERR_CUDA;
}
