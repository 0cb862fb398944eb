// split_harness.cu -- a host build of the decode launches' split planning,
// for CPU tests: the split count of the KV-cache decode and the shares of
// the MLA latent decode, with the workspace sizes that follow from them.
//
// The library's sources are compiled into this program whole, so the
// functions under test are the launches' own: decode_splits,
// decode_split_bytes, decode_workspace_bytes (cache_decode.cu) and
// mla::plan, mla_decode_workspace_bytes (mla_decode.cu).  The two symbols
// those sources take from the rest of the library are defined below; the
// launch paths that would use them are never called.
//
// Input: one query per line on stdin; output: one line per query.
//   dec  k w Hq Hkv d batch max_text
//        "splits split_bytes ws_bytes"
//   mla  k w H batch max_text
//        "tc mt groups splits per ws_bytes"
#include <cstdio>
#include <cstring>
#include <string>

#include "../kv_cache_compression_ksa_b200/csrc/cache_decode.cu"
#include "../kv_cache_compression_ksa_b200/csrc/mla_decode.cu"

extern "C" int64_t ksa_cache_slots(const ksa_params *, int64_t) { return -1; }

namespace ksa {
int sm_count() { return 148; }
namespace mla {
int launch_mla_tc(const Args &, cudaStream_t) { return KSA_ERR_UNSUPPORTED; }
}  // namespace mla
}  // namespace ksa

using namespace ksa;

int main()
{
    char mode[16];
    while (std::scanf("%15s", mode) == 1) {
        if (!std::strcmp(mode, "dec")) {
            int k, w, Hq, Hkv, d, batch;
            long long max_text;
            if (std::scanf("%d %d %d %d %d %d %lld", &k, &w, &Hq, &Hkv, &d, &batch, &max_text) != 7) return 1;
            ksa_params p;
            std::memset(&p, 0, sizeof(p));
            p.k = k; p.w = w; p.num_q_heads = Hq; p.num_kv_heads = Hkv; p.head_dim = d;
            std::printf("%d %zu %zu\n", decode_splits(&p, batch, max_text), decode_split_bytes(&p, batch),
                        decode_workspace_bytes(&p, batch, max_text));
        } else if (!std::strcmp(mode, "mla")) {
            int k, w, H, batch;
            long long max_text;
            if (std::scanf("%d %d %d %d %lld", &k, &w, &H, &batch, &max_text) != 5) return 1;
            ksa_mla_params p;
            std::memset(&p, 0, sizeof(p));
            p.k = k; p.w = w; p.num_heads = H; p.kv_lora_rank = 512; p.rope_dim = 64;
            const mla::Plan P = mla::plan(&p, batch, max_text);
            std::printf("%d %d %d %d %lld %zu\n", P.tc ? 1 : 0, P.mt, P.groups, P.splits, (long long)P.per,
                        mla_decode_workspace_bytes(&p, batch, max_text));
        } else {
            return 1;
        }
        std::fflush(stdout);
    }
    return 0;
}
