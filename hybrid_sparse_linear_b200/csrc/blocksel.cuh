// Block-wide exact selection of the K largest 64-bit keys (selection keys pack an orderable score
// above an inverted block index, so keys are distinct and larger = better).  Used by the decode
// step (span lists, group merge) and by the prefill block selection (pilot seeds).
#pragma once

#include "common.cuh"

namespace sala {

struct RadixSelSmem {
    unsigned hist[256];
    int d, above, eq, nvalid;
};

// Radix select over the E keys each of 256 threads holds (thread index t; key 0 = none): finds the
// K-th largest nonzero key one byte at a time from the top, stopping as soon as the keys sharing
// the resolved prefix are exactly the ones still needed.  On return,
//     winner(key) = key != 0 && (key & mask) >= prefix
// picks exactly min(K, #nonzero) keys.  sync() must be a barrier over the 256 threads.  Keys that
// share their high bytes (nearby scores) would serialize shared-memory atomics on one bin, so the
// lanes holding the same digit add once, through their leader.
template <int E, typename Sync>
__device__ __forceinline__ void radix_kth(const uint64_t (&key)[E], int K, RadixSelSmem& s, uint64_t& prefix,
                          uint64_t& mask, int t, Sync sync) {
    const int lane = t & 31, warp = t >> 5;
    int nv = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) nv += key[e] != 0ull;
    if (t == 0) s.nvalid = 0;
    sync();
    nv = __reduce_add_sync(0xffffffffu, nv);
    if (lane == 0 && nv) atomicAdd(&s.nvalid, nv);
    sync();
    prefix = 0;
    mask = 0;
    if (s.nvalid <= K) {  // every nonzero key wins
        prefix = 1;
        mask = ~0ull;
        return;
    }
    int krem = K;
    for (int shift = 56; shift >= 0; shift -= 8) {
        s.hist[t] = 0;
        sync();
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const bool m = key[e] && (key[e] & mask) == prefix;
            if (!__any_sync(0xffffffffu, m)) continue;
            const unsigned dig = m ? (unsigned)((key[e] >> shift) & 255u) : 256u;
            const unsigned peers = __match_any_sync(0xffffffffu, dig);
            if (m && lane == __ffs(peers) - 1) atomicAdd(&s.hist[dig], (unsigned)__popc(peers));
        }
        sync();
        if (warp == 0) {
            // lane l holds bins 255-8l .. 248-8l (descending order)
            int cnt[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cnt[i] = (int)s.hist[255 - 8 * lane - i];
                sum += cnt[i];
            }
            int incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            const int excl = incl - sum;
            if (excl < krem && krem <= incl) {
                int run = excl;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (run + cnt[i] >= krem) {
                        s.d = 255 - 8 * lane - i;
                        s.above = run;
                        s.eq = cnt[i];
                        break;
                    }
                    run += cnt[i];
                }
            }
        }
        sync();
        krem -= s.above;
        prefix |= (uint64_t)s.d << shift;
        mask |= 0xFFull << shift;
        if (s.eq == krem) break;  // every key with this prefix is a winner
    }
}

}  // namespace sala
