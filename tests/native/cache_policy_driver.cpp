// Drives the expert cache's placement policy (host code only) from commands
// on standard input, for the CPU tests:
//   init E R            -> (nothing)
//   admit n e1 .. en    -> "ok c" then c lines "expert slot", or "full"
//   prefetch n e1 .. en -> "ok c" then c lines "expert slot"
//   pin reserve n e1 .. en -> "ok" / "refused"
//   table               -> "slots s0 .. s(E-1)" (slot of each expert, -1 absent)
//   stats               -> "hits misses" then "uses u0 .. u(E-1)"
#include <cstdio>
#include <iostream>
#include <string>
#include <vector>

#include "../../int4_expert_ffn_router_b200/csrc/expert_cache.h"

int main() {
    coli::ExpertCache c;
    std::string cmd;
    auto read_ids = [](int n) {
        std::vector<int32_t> v(n);
        for (auto& x : v) std::cin >> x;
        return v;
    };
    while (std::cin >> cmd) {
        if (cmd == "init") {
            int E, R;
            std::cin >> E >> R;
            c.init(E, R);
        } else if (cmd == "admit" || cmd == "prefetch") {
            int n;
            std::cin >> n;
            auto ids = read_ids(n);
            std::vector<std::pair<int, int>> copies;
            bool ok = true;
            if (cmd == "admit") ok = c.admit(ids.data(), n, &copies);
            else c.prefetch(ids.data(), n, &copies);
            if (!ok) {
                std::printf("full\n");
                continue;
            }
            std::printf("ok %zu\n", copies.size());
            for (auto& p : copies) std::printf("%d %d\n", p.first, p.second);
        } else if (cmd == "pin") {
            int reserve, n;
            std::cin >> reserve >> n;
            auto ids = read_ids(n);
            std::printf(c.pin(ids.data(), n, reserve) ? "ok\n" : "refused\n");
        } else if (cmd == "table") {
            std::printf("slots");
            for (int e = 0; e < c.E; ++e) std::printf(" %d", c.slot(e));
            std::printf("\n");
        } else if (cmd == "stats") {
            std::printf("%lld %lld\nuses", (long long)c.hits, (long long)c.misses);
            for (int e = 0; e < c.E; ++e) std::printf(" %lld", (long long)c.uses[e]);
            std::printf("\n");
        }
        std::fflush(stdout);
    }
    return 0;
}
