// Concurrency check of the FFN-service mailbox (afd_ffn_mailbox_*), built with ThreadSanitizer by
// tests/test_service_tsan.py on the CPU.  Two producer threads own two slots each and post
// micro-batches; one consumer thread takes them in post order, checks the input pattern, writes
// the output and completes the slot (every seventh one as failed).  Producers check every output.
// The layer entry points the serving loop links against are stubs here: the loop is not started.
#include "afd_ffn.h"

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <thread>
#include <vector>

extern "C" {
int afd_ffn_forward(afd_ffn_handle*, const void*, int32_t, void*, void*) { return AFD_ERR_UNSUPPORTED; }
int afd_ffn_get_info(const afd_ffn_handle*, afd_ffn_cfg*, int32_t*) { return AFD_ERR_INVALID_ARG; }
int afd_ffn_last_cuda_error(const afd_ffn_handle*) { return 0; }
int afd_ffn_get_error(afd_ffn_handle*) { return AFD_OK; }
}

namespace {

constexpr int kSlots = 4, kTmax = 8, kH = 16, kRounds = 400;
std::atomic<int> failures{0};

void check(bool ok, const char* what, int a, int b) {
  if (!ok) {
    if (failures.fetch_add(1) < 10) std::fprintf(stderr, "FAIL %s (%d, %d)\n", what, a, b);
  }
}

uint16_t pattern(int slot, int round, int i) { return static_cast<uint16_t>(slot * 7919 + round * 31 + i); }

void producer(afd_ffn_mailbox* mb, int first_slot) {
  for (int r = 0; r < kRounds; ++r) {
    for (int s = first_slot; s < first_slot + 2; ++s) {
      if (r > 0) {
        const int st = afd_ffn_mailbox_wait(mb, s, 5000000);
        const int prev = r - 1;
        const int T = 1 + (s + prev) % kTmax;
        const bool failed = ((s + prev) % 7) == 0;
        check(st == (failed ? AFD_ERR_CUDA : AFD_OK), "wait status", s, st);
        if (st == AFD_OK) {
          const uint16_t* out = static_cast<const uint16_t*>(afd_ffn_mailbox_output(mb, s));
          for (int i = 0; i < T * kH; ++i) check(out[i] == static_cast<uint16_t>(pattern(s, prev, i) ^ 0xffff), "output", s, i);
        }
      }
      const int T = 1 + (s + r) % kTmax;
      uint16_t* in = static_cast<uint16_t*>(afd_ffn_mailbox_input(mb, s));
      for (int i = 0; i < T * kH; ++i) in[i] = pattern(s, r, i);
      check(afd_ffn_mailbox_post(mb, s, T) == AFD_OK, "post", s, r);
    }
  }
  for (int s = first_slot; s < first_slot + 2; ++s) afd_ffn_mailbox_wait(mb, s, 5000000);
}

void consumer(afd_ffn_mailbox* mb, int total) {
  std::vector<int> round(kSlots, 0);
  for (int n = 0; n < total; ++n) {
    int32_t slot = -1, T = -1;
    const int st = afd_ffn_mailbox_take(mb, &slot, &T, 5000000);
    check(st == AFD_OK, "take", n, st);
    if (st != AFD_OK) return;
    const int r = round[slot]++;
    check(T == 1 + (slot + r) % kTmax, "T", slot, T);
    const uint16_t* in = static_cast<const uint16_t*>(afd_ffn_mailbox_input(mb, slot));
    uint16_t* out = static_cast<uint16_t*>(afd_ffn_mailbox_output(mb, slot));
    for (int i = 0; i < T * kH; ++i) {
      check(in[i] == pattern(slot, r, i), "input", slot, i);
      out[i] = static_cast<uint16_t>(in[i] ^ 0xffff);
    }
    const bool fail = ((slot + r) % 7) == 0;
    check(afd_ffn_mailbox_complete(mb, slot, fail ? AFD_ERR_CUDA : AFD_OK) == AFD_OK, "complete", slot, r);
  }
}

}  // namespace

int main() {
  afd_ffn_mailbox* mb = nullptr;
  if (afd_ffn_mailbox_create(kSlots, kTmax, kH, 0, &mb) != AFD_OK) return 2;
  std::thread c(consumer, mb, kSlots * kRounds);
  std::thread p0(producer, mb, 0), p1(producer, mb, 2);
  p0.join();
  p1.join();
  c.join();
  int32_t slot = 0, T = 0;
  check(afd_ffn_mailbox_take(mb, &slot, &T, 1000) == AFD_ERR_TIMEOUT, "nothing left", 0, 0);
  afd_ffn_mailbox_destroy(mb);
  std::printf("served %d micro-batches, %d failures\n", kSlots * kRounds, failures.load());
  return failures.load() == 0 ? 0 : 1;
}
