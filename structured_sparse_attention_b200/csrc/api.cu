// api.cu -- diagnostics shared by every entry point of libssa.
#include <stdarg.h>
#include <stdio.h>

#include <atomic>

#include "common.cuh"

namespace ssa {

static thread_local char g_last_error[512] = "";
static std::atomic<int64_t> g_wait_limit_ns{2000000000LL};

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
}

int64_t wait_limit_ns() { return g_wait_limit_ns.load(); }

}  // namespace ssa

extern "C" const char *ssa_last_error(void) { return ssa::g_last_error; }

extern "C" int ssa_version(void) { return 100; }

extern "C" int64_t ssa_set_wait_limit_ns(int64_t ns) {
    if (ns < 0) ns = 0;
    return ssa::g_wait_limit_ns.exchange(ns);
}
