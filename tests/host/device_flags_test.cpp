// Host-side check of ds::DeviceFlags, the per-device "done once" record the
// library keeps for each kernel's shared-memory attribute and for the
// no-alloc scratch address: a step done with one device current must not
// count as done for another.  Built and run by tests/test_host_units.py.
#include <cstdio>
#include <thread>
#include <vector>

#include "ds_internal.h"

static int failures = 0;
#define CHECK(c)                                                        \
    do {                                                                \
        if (!(c)) {                                                     \
            std::printf("FAILED: %s (line %d)\n", #c, __LINE__);        \
            ++failures;                                                 \
        }                                                               \
    } while (0)

int main()
{
    ds::DeviceFlags f;
    for (int d = -2; d < 70; ++d)
        CHECK(!f.has(d));
    f.set(0);
    CHECK(f.has(0));
    CHECK(!f.has(1));                 // device 1 still needs its own set-up
    f.set(5);
    CHECK(f.has(5) && f.has(0) && !f.has(4) && !f.has(6));
    f.set(63);
    CHECK(f.has(63));
    f.set(64);                        // ids past 63 are never recorded:
    CHECK(!f.has(64));                // such a device redoes the step each call
    f.set(-1);
    CHECK(!f.has(-1));

    // concurrent first calls on different devices keep every bit
    ds::DeviceFlags g;
    std::vector<std::thread> ts;
    for (int d = 0; d < 64; ++d)
        ts.emplace_back([&g, d] { g.set(d); });
    for (auto &t : ts)
        t.join();
    for (int d = 0; d < 64; ++d)
        CHECK(g.has(d));
    if (failures == 0)
        std::printf("ok\n");
    return failures == 0 ? 0 : 1;
}
