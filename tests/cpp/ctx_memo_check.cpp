// Host-only check of the per-context memo (bit_nf4_quantized_13_b200/csrc/
// ctx_memo.h) that the library uses for its one-time set-up: kernel
// attributes, occupancy answers and the device address of its built-in
// scratch array.  A context id stands for a CUDA context; a device reset
// gives the same device a new id.  Exit status 0 when every check holds.
#include <stdio.h>

#include <atomic>
#include <thread>
#include <vector>

#include "ctx_memo.h"

static int failures = 0;
#define CHECK(c)                                                   \
    do {                                                           \
        if (!(c)) {                                                \
            fprintf(stderr, "check failed line %d: %s\n", __LINE__, #c); \
            ++failures;                                            \
        }                                                          \
    } while (0)

int main() {
    using qlora::ContextMemo;
    {   // one lookup per context; a reset (new id) looks up again
        ContextMemo<void*> memo;
        int fills = 0;
        char a, b;
        void* where = &a;
        auto fill = [&](void** p) { ++fills; *p = where; return true; };
        void* got = nullptr;
        CHECK(memo.get(101, &got, fill) && got == &a && fills == 1);
        CHECK(memo.get(101, &got, fill) && got == &a && fills == 1);
        where = &b;  // the module reloaded at another address after a reset
        CHECK(memo.get(102, &got, fill) && got == &b && fills == 2);
        CHECK(memo.get(101, &got, fill) && got == &a && fills == 2);  // the old context's own entry
        CHECK(memo.size() == 2);
    }
    {   // a failed set-up is not remembered
        ContextMemo<int> memo;
        int calls = 0;
        int v = -1;
        CHECK(!memo.get(7, &v, [&](int* p) { ++calls; *p = 1; return false; }));
        CHECK(memo.size() == 0);
        CHECK(memo.get(7, &v, [&](int* p) { ++calls; *p = 5; return true; }) && v == 5 && calls == 2);
    }
    {   // more contexts than slots: the oldest entries make room, none is wrong
        ContextMemo<int, 4> memo;
        int fills = 0;
        for (uint64_t id = 1; id <= 10; ++id) {
            int v = 0;
            CHECK(memo.get(id, &v, [&](int* p) { ++fills; *p = static_cast<int>(id * 3); return true; }));
            CHECK(v == static_cast<int>(id * 3));
        }
        CHECK(fills == 10 && memo.size() == 4);
        int v = 0;
        CHECK(memo.get(10, &v, [&](int* p) { ++fills; *p = -1; return true; }) && v == 30 && fills == 10);
        CHECK(memo.get(1, &v, [&](int* p) { ++fills; *p = 3; return true; }) && v == 3 && fills == 11);
    }
    {   // concurrent first calls from several threads fill once per context
        ContextMemo<int> memo;
        std::atomic<int> fills{0};
        std::vector<std::thread> th;
        for (int t = 0; t < 8; ++t)
            th.emplace_back([&, t] {
                for (int i = 0; i < 1000; ++i) {
                    int v = 0;
                    const uint64_t id = 1000 + (i + t) % 3;
                    memo.get(id, &v, [&](int* p) { fills.fetch_add(1); *p = static_cast<int>(id); return true; });
                    if (v != static_cast<int>(id)) ++failures;
                }
            });
        for (auto& x : th) x.join();
        CHECK(fills.load() == 3);
    }
    if (failures == 0) printf("ctx_memo: all checks passed\n");
    return failures == 0 ? 0 : 1;
}
