// Launch-configuration overrides for benchmark sweeps: the QOQ_FORCE_CONFIG
// environment variable, read once per process. It changes only how a problem
// is tiled and launched, never what is computed, and size queries see the
// same override as launches.
//
//   QOQ_FORCE_CONFIG="tok=64,cps=1"
//     tok=16|32|64|128|256   token tile (MMA N) for every GEMM
//     cps=1|2                CTAs per SM of the decode kernel (token tiles <= 64)
//     fuse=0|1               qoq_w4a8_linear: quantise the activations inside
//                            the decode GEMM's launch (1) or with the separate
//                            quantiser first (0)
//     kvt=1..8               KV4 attention: 64-token tiles per warp (sets the
//                            tokens per CTA to 256 * kvt)
//     aqt=128|256|512        activation quantiser: threads per CTA
//     aq2=1|2                activation quantiser: the two-pass form (1) or the
//                            row in registers where it fits (2) at every shape
//     lateck=1..10000        GEMM kernels: every contributor to a split
//                            tile arrives this many microseconds late (a
//                            sleep), so that owners arrive first and the last
//                            contributor finishes each tile (a test of that path)
//     prs=1|2|3              RMSNorm producer, rows of up to 4096: keep the
//                            normalised row in registers (1), form it again
//                            for the codes (2), or stage the input row in
//                            shared memory and loop over it (3)
//     pst=1|2                SiLU-gated producer, rows above 8192: the narrower
//                            (1) or the wider (2) of its two CTA shapes
// Unknown keys and values are ignored.
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "qoq_internal.h"

namespace qoq {

const ForcedConfig &forced_config() {
    static ForcedConfig cfg;
    static std::once_flag once;
    std::call_once(once, [] {
        const char *env = std::getenv("QOQ_FORCE_CONFIG");
        if (env == nullptr) return;
        const char *p = env;
        while (*p) {
            const char *end = std::strchr(p, ',');
            const size_t len = end ? (size_t)(end - p) : std::strlen(p);
            int v = 0;
            if (len > 4 && std::strncmp(p, "tok=", 4) == 0) {
                v = std::atoi(p + 4);
                if (v == 16 || v == 32 || v == 64 || v == 128 || v == 256) cfg.tok = v;
            } else if (len > 4 && std::strncmp(p, "cps=", 4) == 0) {
                v = std::atoi(p + 4);
                if (v == 1 || v == 2) cfg.cps = v;
            } else if (len > 7 && std::strncmp(p, "lateck=", 7) == 0) {
                v = std::atoi(p + 7);
                if (v >= 1 && v <= 10000) cfg.lateck = v;
            } else if (len > 4 && std::strncmp(p, "aq2=", 4) == 0) {
                v = std::atoi(p + 4);
                if (v == 1 || v == 2) cfg.aq2 = v;
            } else if (len > 4 && std::strncmp(p, "prs=", 4) == 0) {
                v = std::atoi(p + 4);
                if (v >= 1 && v <= 3) cfg.prs = v;
            } else if (len > 4 && std::strncmp(p, "pst=", 4) == 0) {
                v = std::atoi(p + 4);
                if (v == 1 || v == 2) cfg.pst = v;
            } else if (len > 4 && std::strncmp(p, "aqt=", 4) == 0) {
                v = std::atoi(p + 4);
                if (v == 128 || v == 256 || v == 512) cfg.aqt = v;
            } else if (len > 4 && std::strncmp(p, "kvt=", 4) == 0) {
                v = std::atoi(p + 4);
                if (v >= 1 && v <= 8) cfg.kvt = v;
            } else if (len > 5 && std::strncmp(p, "fuse=", 5) == 0) {
                v = std::atoi(p + 5);
                if (v == 0 || v == 1) cfg.fuse = v + 1;
            }
            if (!end) break;
            p = end + 1;
        }
    });
    return cfg;
}

}  // namespace qoq
