// Host replay of the persistent factorisation's task queue (chol_persist_kernel).
//
// The kernel's CTAs take tasks from one counter in queue order, and a task
// may wait on counters other tasks publish.  Every wait ends, with any number
// of resident CTAs, if each task's waits are met by tasks earlier in the
// queue.  This program walks the queue in order with the kernel's own task
// decoder, checks every wait against what the earlier tasks published, checks
// that every tile receives its panels' updates in panel order, and checks the
// final counts.  It runs no GPU code (built as PTX only, never launched).
//
// Usage: replay_factorisation  -> exit 0 and "ok <shapes>" when every width
// n = 128 nblk, nblk = 3 .. 63, passes; exit 1 with the first failure.
#include "../post_weight_quantization_25_b200/csrc/cholesky.cu"

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

static int fail(int n, int t, const char* what) {
  std::printf("n=%d task %d: %s\n", n, t, what);
  return 1;
}

static int check(int n) {
  const int nblk = n / kPanel;
  const int T = cp_total(nblk, n);
  // the kernel's counters: panels applied per tile, apply chunks per row
  // block and panel parity, update tasks per panel, diagonal blocks done
  std::vector<long> tile((size_t)nblk * nblk, 0), vdone(2 * (size_t)nblk, 0), tdone(nblk, 0),
      ddone(nblk, 0);
  for (int t = 0; t < T; ++t) {
    const CpTask k = cp_decode(nblk, n, t);
    const int p = k.p;
    if (p < 0 || p >= nblk) return fail(n, t, "panel out of range");
    if (k.kind == 0 || k.kind == 1) {
      int R0 = 0, R1 = 0;
      if (k.kind == 1) {
        if (k.k < 0 || k.k >= n / 32) return fail(n, t, "apply chunk out of range");
        const int nA = n - (p + 1) * kPanel, v0 = 32 * k.k, v1 = v0 + 31;
        R0 = v0 < nA ? p + 1 + v0 / kPanel : (v0 - nA) / kPanel;
        R1 = v1 < nA ? p + 1 + v1 / kPanel : (v1 - nA) / kPanel;
        if (R0 < 0 || R1 >= nblk || R0 != R1) return fail(n, t, "apply rows out of range");
        if (!ddone[p]) return fail(n, t, "apply before its diagonal block");
        for (int R = R0; R <= R1; ++R)
          if (tile[(size_t)R * nblk + p] < (R > p ? p : p - R))
            return fail(n, t, "apply before its rows have the earlier panels");
      } else {
        if (tile[(size_t)p * nblk + p] < p) return fail(n, t, "diagonal block before its updates");
        if (ddone[p]) return fail(n, t, "second diagonal task of a panel");
      }
      if (p >= 2 && tdone[p - 2] < cp_update_tasks(nblk, p - 2))
        return fail(n, t, "buffers reused before panel p - 2's updates are done");
      if (k.kind == 0) {
        ddone[p] = 1;
      } else {
        ++vdone[(size_t)(p & 1) * nblk + R0];
      }
      continue;
    }
    if (k.kind != 2) return fail(n, t, "unknown task kind");
    const int R = k.R;
    if (R < 0 || R >= nblk || k.c0 <= p || k.c1 > nblk || k.c0 >= k.c1 || k.c1 - k.c0 > kCpChunk)
      return fail(n, t, "update tiles out of range");
    const long vneed = 4 * (p / 2 + 1);
    if (vdone[(size_t)(p & 1) * nblk + R] < vneed) return fail(n, t, "update before its P rows");
    for (int S = k.c0; S < k.c1; ++S) {
      if (vdone[(size_t)(p & 1) * nblk + S] < vneed) return fail(n, t, "update before its Q rows");
      const long want = R >= S ? p : p - R;
      const long have = tile[(size_t)R * nblk + S];
      if (have < want) return fail(n, t, "update before the tile has the earlier panels");
      if (have > want) return fail(n, t, "tile updated out of panel order");
      tile[(size_t)R * nblk + S] = want + 1;
    }
    ++tdone[p];
  }
  for (int p = 0; p < nblk; ++p) {
    if (!ddone[p]) return fail(n, T, "a diagonal block never ran");
    if (tdone[p] != cp_update_tasks(nblk, p)) return fail(n, T, "update count of a panel");
  }
  // tile (R, S) of the lower part takes panels 0 .. S - 1, of the
  // transposed part panels R .. S - 1
  for (int R = 0; R < nblk; ++R)
    for (int S = 0; S < nblk; ++S)
      if (tile[(size_t)R * nblk + S] != (R >= S ? S : S - R)) return fail(n, T, "final tile count");
  return 0;
}

int main() {
  int shapes = 0;
  for (int nblk = 3; nblk < 64; ++nblk, ++shapes)
    if (check(nblk * kPanel)) return 1;
  std::printf("ok %d\n", shapes);
  return 0;
}
