// Host replay of the persistent sweep's task queue (sweep_persist_kernel).
//
// The same argument as for the factorisation: every wait ends, with any
// number of resident CTAs, if each task's waits are met by tasks earlier in
// the queue.  This program walks the queue in order with the kernel's own
// task decoder and checks four things:
// - a sweep task of block s finds tile s, and every tile of a group ruler
//   wider than a block that starts at s, repaired by blocks 0 .. s - 1;
// - an update by block b finds block b swept for all of its rows;
// - every tile receives the blocks' updates in block order;
// - at the end tile c holds blocks 0 .. c - 1 and every block is swept.
// It runs no GPU code (built as PTX only, never launched).
//
// Usage: replay_sweep  -> exit 0 and "ok <shapes>" when every shape passes.
#include "../post_weight_quantization_25_b200/csrc/sweep.cu"

#include <cstdio>
#include <vector>

// the library functions the included source refers to (never called here)
namespace gptq {
void note_launch() {}
int num_sms() { return 148; }
bool make_tma_2d(CUtensorMap*, const void*, bool, int64_t, int64_t, int64_t, uint32_t, uint32_t) {
  return false;
}
WaitGate current_wait_gate() { return WaitGate{nullptr, 0}; }
bool SideEvents::create() { return false; }
SideEvents::~SideEvents() {}
}  // namespace gptq

using namespace gptq;

static int fail(const SweepPersistArgs& a, int t, const char* what) {
  std::printf("RB=%d nb=%d gw=%d task %d: %s\n", a.RB, a.nb, a.gw, t, what);
  return 1;
}

static int check(int RB, int nb, int gw) {
  SweepPersistArgs a{};
  a.RB = RB;
  a.nb = nb;
  a.gw = gw;
  const int T = sp_total(a);
  std::vector<long> swept(RB, 0), applied((size_t)RB * nb, 0);
  std::vector<char> seen((size_t)RB * nb * kSpSlices, 0);
  for (int t = 0; t < T; ++t) {
    const SpTask k = sp_decode(a, t);
    const int R = k.R, s = k.s;
    if (R < 0 || R >= RB || s < 0 || s >= nb) return fail(a, t, "task out of range");
    if (k.kind == 0) {
      if (k.slice < 0 || k.slice >= kSpSlices) return fail(a, t, "slice out of range");
      char& once = seen[((size_t)R * nb + s) * kSpSlices + k.slice];
      if (once) return fail(a, t, "slice swept twice");
      once = 1;
      int c_hi = s + 1;
      if (gw > 1 && s % gw == 0) c_hi = std::min(nb, s + gw);
      for (int c = s; c < c_hi; ++c)
        if (applied[(size_t)R * nb + c] < s) return fail(a, t, "sweep before its columns are repaired");
      ++swept[R];
      continue;
    }
    if (k.kind != 1) return fail(a, t, "unknown task kind");
    if (k.c0 <= s || k.c1 > nb || k.c0 >= k.c1 || k.c1 - k.c0 > kSpChunk)
      return fail(a, t, "update tiles out of range");
    if (swept[R] < (long)kSpSlices * (s + 1)) return fail(a, t, "update before its block is swept");
    for (int c = k.c0; c < k.c1; ++c) {
      long& have = applied[(size_t)R * nb + c];
      if (have < s) return fail(a, t, "update before the tile has the earlier blocks");
      if (have > s) return fail(a, t, "tile updated out of block order");
      have = s + 1;
    }
  }
  for (int R = 0; R < RB; ++R) {
    if (swept[R] != (long)kSpSlices * nb) return fail(a, T, "a slice was never swept");
    for (int c = 0; c < nb; ++c)
      if (applied[(size_t)R * nb + c] != c) return fail(a, T, "final tile count");
  }
  return 0;
}

int main() {
  int shapes = 0;
  const int rbs[] = {1, 2, 3, 5, 32, 64};
  const int gws[] = {1, 2, 3, 4, 8};
  for (int RB : rbs)
    for (int nb = 2; nb < 64; ++nb)
      for (int gw : gws) {
        if (check(RB, nb, gw)) return 1;
        ++shapes;
      }
  std::printf("ok %d\n", shapes);
  return 0;
}
