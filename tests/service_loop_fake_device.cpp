// The FFN serving loop (afd_ffn_service_*) on the CPU, built with ThreadSanitizer by
// tests/test_service_tsan.py.  The CUDA runtime calls the service makes are defined here as a
// synchronous fake device (copies are memcpy, events complete ~50 us after they are recorded),
// and the layer is a stub that writes out = in ^ 0xffff.  This runs the loop thread, the
// completer thread and the producer against each other: in-order service of many micro-batches,
// a failing layer call and the status it leaves, and stop with slots still posted.
#include "afd_ffn.h"

#include <cuda_runtime.h>
#include <time.h>

#include <atomic>
#include <chrono>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <thread>

namespace {

int64_t now_ns() {
  timespec ts;
  clock_gettime(CLOCK_MONOTONIC, &ts);
  return static_cast<int64_t>(ts.tv_sec) * 1000000000LL + ts.tv_nsec;
}

struct FakeEvent {
  std::atomic<int64_t> done_at{0};   // 0: never recorded
};

struct FakeHandle {
  afd_ffn_cfg cfg;
  std::atomic<int> fail_T{-1};       // a layer call with this T fails
  std::atomic<int> delay_us{0};      // each layer call takes this long
};

std::atomic<int> failures{0};

void check(bool ok, const char* what, long a, long b) {
  if (!ok && failures.fetch_add(1) < 10) std::fprintf(stderr, "FAIL %s (%ld, %ld)\n", what, a, b);
}

}  // namespace

// ---- fake CUDA runtime (only what the service calls)
extern "C" {
cudaError_t cudaHostAlloc(void** p, size_t n, unsigned int) { *p = std::aligned_alloc(64, (n + 63) / 64 * 64); return *p ? cudaSuccess : cudaErrorMemoryAllocation; }
cudaError_t cudaFreeHost(void* p) { std::free(p); return cudaSuccess; }
cudaError_t cudaMalloc(void** p, size_t n) { *p = std::malloc(n ? n : 1); return *p ? cudaSuccess : cudaErrorMemoryAllocation; }
cudaError_t cudaFree(void* p) { std::free(p); return cudaSuccess; }
cudaError_t cudaSetDevice(int) { return cudaSuccess; }
cudaError_t cudaGetDevice(int* d) { *d = 0; return cudaSuccess; }
cudaError_t cudaGetLastError(void) { return cudaSuccess; }
cudaError_t cudaStreamCreateWithFlags(cudaStream_t* s, unsigned int) { *s = reinterpret_cast<cudaStream_t>(new int(0)); return cudaSuccess; }
cudaError_t cudaStreamDestroy(cudaStream_t s) { delete reinterpret_cast<int*>(s); return cudaSuccess; }
cudaError_t cudaStreamSynchronize(cudaStream_t) { return cudaSuccess; }
cudaError_t cudaStreamWaitEvent(cudaStream_t, cudaEvent_t, unsigned int) { return cudaSuccess; }
cudaError_t cudaEventCreate(cudaEvent_t* e) { *e = reinterpret_cast<cudaEvent_t>(new FakeEvent); return cudaSuccess; }
cudaError_t cudaEventDestroy(cudaEvent_t e) { delete reinterpret_cast<FakeEvent*>(e); return cudaSuccess; }
cudaError_t cudaEventRecord(cudaEvent_t e, cudaStream_t) {
  reinterpret_cast<FakeEvent*>(e)->done_at.store(now_ns() + 50000);
  return cudaSuccess;
}
cudaError_t cudaEventQuery(cudaEvent_t e) {
  const int64_t t = reinterpret_cast<FakeEvent*>(e)->done_at.load();
  return (t == 0 || now_ns() >= t) ? cudaSuccess : cudaErrorNotReady;
}
cudaError_t cudaEventElapsedTime(float* ms, cudaEvent_t a, cudaEvent_t b) {
  *ms = static_cast<float>(reinterpret_cast<FakeEvent*>(b)->done_at.load() - reinterpret_cast<FakeEvent*>(a)->done_at.load()) / 1e6f;
  return cudaSuccess;
}
cudaError_t cudaMemcpyAsync(void* dst, const void* src, size_t n, cudaMemcpyKind, cudaStream_t) {
  std::memcpy(dst, src, n);
  return cudaSuccess;
}

// ---- the layer entry points the service links against
int afd_ffn_get_info(const afd_ffn_handle* h, afd_ffn_cfg* cfg, int32_t* device) {
  if (!h) return AFD_ERR_INVALID_ARG;
  if (cfg) *cfg = reinterpret_cast<const FakeHandle*>(h)->cfg;
  if (device) *device = 0;
  return AFD_OK;
}
int afd_ffn_forward(afd_ffn_handle* h, const void* in, int32_t T, void* out, void*) {
  FakeHandle* f = reinterpret_cast<FakeHandle*>(h);
  if (T == f->fail_T.load()) return AFD_ERR_UNSUPPORTED;
  if (const int d = f->delay_us.load()) std::this_thread::sleep_for(std::chrono::microseconds(d));
  const uint16_t* a = static_cast<const uint16_t*>(in);
  uint16_t* b = static_cast<uint16_t*>(out);
  for (int64_t i = 0; i < static_cast<int64_t>(T) * f->cfg.H; ++i) b[i] = static_cast<uint16_t>(a[i] ^ 0xffff);
  return AFD_OK;
}
int afd_ffn_last_cuda_error(const afd_ffn_handle*) { return 0; }
int afd_ffn_get_error(afd_ffn_handle*) { return AFD_OK; }
}

namespace {

constexpr int kSlots = 3, kTmax = 8, kH = 16;

uint16_t pattern(long n, int i) { return static_cast<uint16_t>(n * 131 + i); }

afd_ffn_handle* as_handle(FakeHandle* f) { return reinterpret_cast<afd_ffn_handle*>(f); }

void write_input(afd_ffn_mailbox* mb, int slot, long n, int T) {
  uint16_t* in = static_cast<uint16_t*>(afd_ffn_mailbox_input(mb, slot));
  for (int i = 0; i < T * kH; ++i) in[i] = pattern(n, i);
}

void check_output(afd_ffn_mailbox* mb, int slot, long n, int T) {
  const uint16_t* out = static_cast<const uint16_t*>(afd_ffn_mailbox_output(mb, slot));
  for (int i = 0; i < T * kH; ++i) check(out[i] == static_cast<uint16_t>(pattern(n, i) ^ 0xffff), "output", n, i);
}

// many micro-batches through every slot, each checked
void in_order_service(FakeHandle* f) {
  afd_ffn_mailbox* mb = nullptr;
  check(afd_ffn_mailbox_create(kSlots, kTmax, kH, 0, &mb) == AFD_OK, "create", 0, 0);
  afd_ffn_service* svc = nullptr;
  check(afd_ffn_service_start(as_handle(f), mb, nullptr, &svc) == AFD_OK, "start", 0, 0);
  afd_ffn_service* second = nullptr;
  check(afd_ffn_service_start(as_handle(f), mb, nullptr, &second) == AFD_ERR_INVALID_ARG, "one loop per mailbox", 0, 0);
  const long total = 600;
  long posted[kSlots] = {-1, -1, -1};
  for (long n = 0; n < total + kSlots; ++n) {
    const int s = static_cast<int>(n % kSlots);
    if (posted[s] >= 0) {
      check(afd_ffn_mailbox_wait(mb, s, 5000000) == AFD_OK, "wait", n, s);
      check_output(mb, s, posted[s], 1 + static_cast<int>(posted[s] % kTmax));
      float ms[5];
      check(afd_ffn_service_slot_timeline(svc, s, ms) == AFD_OK, "timeline", n, s);
      posted[s] = -1;
    }
    if (n < total) {
      const int T = 1 + static_cast<int>(n % kTmax);
      write_input(mb, s, n, T);
      check(afd_ffn_mailbox_post(mb, s, T) == AFD_OK, "post", n, s);
      posted[s] = n;
    }
  }
  afd_ffn_service_stats st;
  check(afd_ffn_service_stop(svc, &st) == AFD_OK, "stop", 0, 0);
  check(st.served == total && st.status == AFD_OK, "stats", static_cast<long>(st.served), st.status);
  afd_ffn_mailbox_destroy(mb);
}

// a failing layer call fails its slot and every later one with the same status
void failure_propagates(FakeHandle* f) {
  afd_ffn_mailbox* mb = nullptr;
  check(afd_ffn_mailbox_create(kSlots, kTmax, kH, 0, &mb) == AFD_OK, "create", 1, 0);
  afd_ffn_service* svc = nullptr;
  f->fail_T.store(5);
  check(afd_ffn_service_start(as_handle(f), mb, nullptr, &svc) == AFD_OK, "start", 1, 0);
  write_input(mb, 0, 0, 3);
  afd_ffn_mailbox_post(mb, 0, 3);
  check(afd_ffn_mailbox_wait(mb, 0, 5000000) == AFD_OK, "before the failure", 0, 0);
  afd_ffn_mailbox_post(mb, 1, 5);
  check(afd_ffn_mailbox_wait(mb, 1, 5000000) == AFD_ERR_UNSUPPORTED, "failing call", 1, 0);
  afd_ffn_mailbox_post(mb, 2, 2);
  check(afd_ffn_mailbox_wait(mb, 2, 5000000) == AFD_ERR_UNSUPPORTED, "after the failure", 2, 0);
  afd_ffn_service_stats st;
  check(afd_ffn_service_stop(svc, &st) == AFD_ERR_UNSUPPORTED, "stop status", st.status, 0);
  check(st.served == 1, "served before the failure", static_cast<long>(st.served), 0);
  f->fail_T.store(-1);
  afd_ffn_mailbox_destroy(mb);
}

// stop while slots are still posted: each completes or fails with AFD_ERR_STOPPED
void stop_with_posted_slots(FakeHandle* f) {
  afd_ffn_mailbox* mb = nullptr;
  check(afd_ffn_mailbox_create(kSlots, kTmax, kH, 0, &mb) == AFD_OK, "create", 2, 0);
  afd_ffn_service* svc = nullptr;
  f->delay_us.store(3000);
  check(afd_ffn_service_start(as_handle(f), mb, nullptr, &svc) == AFD_OK, "start", 2, 0);
  for (int s = 0; s < kSlots; ++s) {
    write_input(mb, s, s, 4);
    afd_ffn_mailbox_post(mb, s, 4);
  }
  std::this_thread::sleep_for(std::chrono::microseconds(500));   // the loop is inside slot 0's layer
  afd_ffn_service_stats st;
  check(afd_ffn_service_stop(svc, &st) == AFD_OK, "stop", 2, 0);
  int ok = 0, stopped = 0;
  for (int s = 0; s < kSlots; ++s) {
    const int r = afd_ffn_mailbox_wait(mb, s, 1000000);
    ok += r == AFD_OK;
    stopped += r == AFD_ERR_STOPPED;
    if (r == AFD_OK) check_output(mb, s, s, 4);
  }
  check(ok + stopped == kSlots, "every slot ended", ok, stopped);
  check(ok >= 1 && stopped >= 1, "one served, the rest stopped", ok, stopped);
  check(st.served == ok, "served count", static_cast<long>(st.served), ok);
  f->delay_us.store(0);
  afd_ffn_mailbox_destroy(mb);
}

}  // namespace

int main() {
  FakeHandle f;
  std::memset(&f.cfg, 0, sizeof(f.cfg));
  f.cfg.T_max = kTmax;
  f.cfg.H = kH;
  in_order_service(&f);
  failure_propagates(&f);
  stop_with_posted_slots(&f);
  std::printf("serving loop: %d failures\n", failures.load());
  return failures.load() == 0 ? 0 : 1;
}
