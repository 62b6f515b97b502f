// Host driver for the kernels' bounded-wait template (csrc/bounded_wait.cuh),
// built and run by tests/test_bounded_wait_cpu.py.  A fake clock advances by
// one per reading and a fake condition becomes true after a given number of
// polls.  Prints one line per case: name, result (0/1), polls made.
#include <cstdio>

#include "bounded_wait.cuh"

struct Case {
  const char* name;
  unsigned long long limit;
  long ready_after;   // polls before ready() returns true; < 0: never
  int abort_at;       // set the abort flag once this many polls were made; < 0: never
  unsigned every;
};

int main() {
  const Case cases[] = {
      {"ready_at_once", 0, 0, -1, 32},
      {"cap0_never_ready", 0, -1, -1, 32},
      {"cap0_never_ready_every16", 0, -1, -1, 16},
      {"ready_before_limit", 1000, 500, -1, 32},
      {"limit_runs_out", 100, -1, -1, 32},
      {"abort_flag", 1ull << 40, -1, 70, 32},
  };
  for (const Case& c : cases) {
    long polls = 0;
    unsigned long long clock = 0;
    int abort_flag = 0;
    const bool ok = moe::bounded_poll(
        [&] {
          ++polls;
          if (c.abort_at >= 0 && polls >= c.abort_at) abort_flag = 1;
          return c.ready_after >= 0 && polls > c.ready_after;
        },
        [&] { return clock++; }, [] {}, &abort_flag, c.limit, c.every);
    std::printf("%s %d %ld\n", c.name, ok ? 1 : 0, polls);
  }
  return 0;
}
