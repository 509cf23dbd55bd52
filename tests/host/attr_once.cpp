// Host test of zha::PerDeviceMax: a fake sequence of launches on two devices
// (the setter counts its calls instead of calling the CUDA runtime).
#include <cstdio>
#include <thread>
#include <vector>

#include "../../tree_indexed_sparse_b200/csrc/zha_attr.h"

static zha::PerDeviceMax<4> rec;

#define CHECK(x)                                                   \
    do {                                                           \
        if (!(x)) {                                                \
            std::printf("FAIL line %d: %s\n", __LINE__, #x);       \
            return 1;                                              \
        }                                                          \
    } while (0)

int main() {
    int calls[6] = {0, 0, 0, 0, 0, 0};
    auto setter = [&](int dev) { return [&, dev](long long) { calls[dev] += 1; return 0; }; };
    // device 0: first launch sets, the same size again does not
    CHECK(rec.raise(0, 100, setter(0)) == 0 && calls[0] == 1);
    CHECK(rec.raise(0, 100, setter(0)) == 0 && calls[0] == 1);
    // device 1 must be set on its own, although device 0 already is
    CHECK(rec.raise(1, 100, setter(1)) == 0 && calls[1] == 1);
    // a larger need raises again; a smaller one does not
    CHECK(rec.raise(0, 200, setter(0)) == 0 && calls[0] == 2);
    CHECK(rec.raise(0, 150, setter(0)) == 0 && calls[0] == 2);
    CHECK(rec.raise(1, 150, setter(1)) == 0 && calls[1] == 2);
    // a failing setter leaves nothing recorded, so the next launch retries
    CHECK(rec.raise(2, 64, [](long long) { return 7; }) == 7);
    CHECK(rec.raise(2, 64, setter(2)) == 0 && calls[2] == 1);
    // a device ordinal past the table sets every time
    CHECK(rec.raise(9, 64, setter(5)) == 0 && rec.raise(9, 64, setter(5)) == 0 && calls[5] == 2);
    // concurrent first launches on one device: set at least once, recorded once
    std::atomic<int> n{0};
    std::vector<std::thread> th;
    for (int i = 0; i < 8; ++i)
        th.emplace_back([&] { rec.raise(3, 300, [&](long long) { n.fetch_add(1); return 0; }); });
    for (auto &t : th) t.join();
    CHECK(n.load() >= 1 && rec.done[3].load() == 300);
    CHECK(rec.raise(3, 300, [&](long long) { n.fetch_add(1000); return 0; }) == 0 && n.load() < 1000);
    std::printf("ok\n");
    return 0;
}
