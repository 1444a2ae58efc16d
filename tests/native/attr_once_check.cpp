// CPU check of the per-(kernel, device) attribute bookkeeping in bl_attr.h:
// a setting runs once per device, a failed setting is retried, keys are kept
// apart, and out-of-range devices are refused.  Prints "ok" on success.
#include <cstdio>

#include "bl_attr.h"

#define CHECK(c)                                                   \
    do {                                                           \
        if (!(c)) {                                                \
            std::printf("FAIL line %d: %s\n", __LINE__, #c);       \
            return 1;                                              \
        }                                                          \
    } while (0)

int main() {
    bl::AttrOnce once;
    int k1 = 0, k2 = 0;
    int calls = 0;
    auto ok = [&] { ++calls; return 0; };
    auto fail = [&] { ++calls; return 7; };

    CHECK(once.ensure(&k1, 0, ok) == 0 && calls == 1);
    CHECK(once.ensure(&k1, 0, ok) == 0 && calls == 1);   // device 0 already set
    CHECK(once.ensure(&k1, 1, ok) == 0 && calls == 2);   // a second device sets it again
    CHECK(once.is_set(&k1, 0) && once.is_set(&k1, 1) && !once.is_set(&k1, 2));
    CHECK(once.ensure(&k2, 1, fail) == 7 && calls == 3); // failure is reported ...
    CHECK(!once.is_set(&k2, 1));
    CHECK(once.ensure(&k2, 1, fail) == 7 && calls == 4); // ... and retried
    CHECK(once.ensure(&k2, 1, ok) == 0 && calls == 5);
    CHECK(once.ensure(&k2, 1, ok) == 0 && calls == 5);
    CHECK(once.ensure(&k1, 63, ok) == 0 && calls == 6);
    CHECK(once.ensure(&k1, 64, ok) == -1 && calls == 6); // outside the table
    CHECK(once.ensure(&k1, -1, ok) == -1 && calls == 6);
    int keys[bl::AttrOnce::kKeys];
    int filled = 0;
    for (int i = 0; i < bl::AttrOnce::kKeys; ++i)
        if (once.ensure(&keys[i], 0, ok) == 0) ++filled;
    CHECK(filled == bl::AttrOnce::kKeys - 2);            // k1 and k2 hold two slots
    std::printf("ok\n");
    return 0;
}
