// attn_tiles.cuh -- the work-tile schedule shared by the attention kernels: tile index ->
// (sequence, KV head, query block, query head), the tile's kept-block list, and the static
// per-worker walk over tiles.
#pragma once

#include "internal.h"
#include "sm100.cuh"

namespace bsa {

// Work tile t -> (b, hk, i, g); tiles are ordered sequence-major, then KV head, then query
// block from the last one down, then the G query heads of the group.
struct Tile {
    int b, h, hk, i, n_tok, nb, n_list, l_begin;
    bool valid;
};

__device__ __forceinline__ Tile decode_tile(const AttnArgs& a, int t) {
    Tile T;
    const int G = a.Hq / a.Hkv;
    const int per_b = a.Hkv * a.nb_max * G;
    T.b = t / per_b;
    int x = t % per_b;
    const int g = x % G;
    x /= G;
    T.i = a.nb_max - 1 - (x % a.nb_max);
    T.hk = x / a.nb_max;
    T.h = T.hk * G + g;
    T.n_tok = a.seqlen[T.b];
    T.nb = (T.n_tok + a.block - 1) / a.block;
    T.valid = T.i < T.nb;
    T.n_list = 0;
    T.l_begin = 0;
    if (T.valid) {
        const int32_t* rp = a.row_ptr + static_cast<int64_t>(T.b) * a.row_ptr_stride +
                            static_cast<int64_t>(T.h) * a.row_ptr_hstride;
        T.l_begin = __ldg(rp + T.i);
        T.n_list = __ldg(rp + T.i + 1) - T.l_begin;
        if (T.n_list < 1 || T.n_list > kMaxBlocks || T.l_begin < 0 ||
            T.l_begin + static_cast<int64_t>(T.n_list) > a.max_k) {
            T.n_list = 0;  // empty or corrupt row pointer: the tile is skipped
        }
    }
    return T;
}

// Physical page of logical page lp (tokens 64*lp ...) of sequence b for a paged K/V load:
// num_pages (a box the TMA reads as zeros) past the end of the sequence; an entry outside
// [0, num_pages) is recorded in `bad` (kDevErrInvalidPage) and read as zeros too.
__device__ __forceinline__ int physical_page(const AttnArgs& a, int b, int lp, int n_tok, unsigned& bad) {
    if (lp * 64 >= n_tok) return a.num_pages;
    const int phys = __ldg(a.page_table + static_cast<int64_t>(b) * a.max_pages + lp);
    if (phys < 0 || phys >= a.num_pages) {
        bad |= kDevErrInvalidPage;
        return a.num_pages;
    }
    return phys;
}

// List entry n of the tile; -1 if out of [0, i] (skipped block: scores all -inf).  The lists
// are per query head (col_idx [B, Hq, max_k]) or, for group-shared selection, per KV head
// (col_idx [B, Hkv, max_k]).
__device__ __forceinline__ int list_entry(const AttnArgs& a, const Tile& T, int n) {
    const int64_t row = a.list_per_group ? static_cast<int64_t>(T.b) * a.Hkv + T.hk
                                         : static_cast<int64_t>(T.b) * a.Hq + T.h;
    const int j = __ldg(a.col_idx + row * a.max_k + T.l_begin + n);
    return (j >= 0 && j <= T.i) ? j : -1;
}

// Entry n of the tile's list as stored (0 for n past the end, which no block uses), and the
// range check of list_entry applied to such a value: the two halves of list_entry for a
// caller that loads entries ahead of their use.
__device__ __forceinline__ int list_entry_raw(const AttnArgs& a, const Tile& T, int n) {
    if (n >= T.n_list) return 0;
    const int64_t row = a.list_per_group ? static_cast<int64_t>(T.b) * a.Hkv + T.hk
                                         : static_cast<int64_t>(T.b) * a.Hq + T.h;
    return __ldg(a.col_idx + row * a.max_k + T.l_begin + n);
}
__device__ __forceinline__ int list_entry_check(const Tile& T, int j) { return (j >= 0 && j <= T.i) ? j : -1; }

// The static tile sequence of one slot: tiles base + s, base + s + stride, ... that are
// non-empty.  Every role walks the same sequence.
struct TileIter {
    int round, s, base, stride, total;
    bool active;
    Tile T;
    __device__ __forceinline__ void init(int s_, int base_, int stride_, int total_) {
        s = s_;
        base = base_;
        stride = stride_;
        total = total_;
        round = 0;
        active = true;
    }
    __device__ __forceinline__ void next(const AttnArgs& a) {
        while (true) {
            const int t = base + s + round * stride;
            ++round;
            if (t >= total) {
                active = false;
                return;
            }
            T = decode_tile(a, t);
            if (T.valid && T.n_list > 0) return;
        }
    }
};

// Dynamic tile schedule.  The producer warp takes the next tile index from the launch's
// counter (a.tile_counter, zeroed before the launch) and hands it to the CTA's other roles
// through a ring in shared memory; -1 means no tile is left.  Tiles are taken in index order
// (sequence, KV head, query block from the last, query head), so the heavy tiles go first and
// each CTA takes the next one when it is free.
constexpr int kTileRing = 4;

struct TileRing {
    uint64_t full[kTileRing], empty[kTileRing];
    int idx[kTileRing];
};

// One thread, before the CTA's first barrier: `consumers` arrivals free a slot.
__device__ __forceinline__ void tile_ring_init(TileRing& r, int consumers) {
    for (int t = 0; t < kTileRing; ++t) {
        mbar_init(&r.full[t], 1);
        mbar_init(&r.empty[t], consumers);
    }
}

// Producer, one thread: publishes, in slot n % kTileRing, the tile of the next counter value
// c < total whose tile to_tile(c) is not empty (or -1 when none is left); t receives it.  The
// counter runs over work units, to_tile maps a unit to the tile index the consumers decode
// (the identity for per-head tiles).  False when the wait for the slot failed (nothing
// published).
struct TileIdentity {
    __device__ __forceinline__ int operator()(int c) const { return c; }
};
template <class ToTile = TileIdentity>
__device__ __forceinline__ bool tile_ring_put(TileRing& r, uint32_t n, const AttnArgs& a, int total, int& t,
                                              volatile int* abort_flag, ToTile to_tile = ToTile()) {
    const uint32_t slot = n % kTileRing;
    if (!mbar_wait(&r.empty[slot], ((n / kTileRing) & 1) ^ 1, abort_flag, a.err)) return false;
    while (true) {
        const int c = atomicAdd(a.tile_counter, 1);
        if (c >= total) {
            t = -1;
            break;
        }
        t = to_tile(c);
        const Tile U = decode_tile(a, t);
        if (U.valid && U.n_list > 0) break;
    }
    r.idx[slot] = t;
    mbar_arrive(&r.full[slot]);
    return true;
}

// Consumer, one thread: the tile in slot n % kTileRing (frees the slot).  1: a tile, 0: none
// left, -1: the wait failed.
__device__ __forceinline__ int tile_ring_get(TileRing& r, uint32_t n, const AttnArgs& a, Tile& T,
                                             volatile int* abort_flag) {
    const uint32_t slot = n % kTileRing;
    if (!mbar_wait(&r.full[slot], (n / kTileRing) & 1, abort_flag, a.err)) return -1;
    const int t = *reinterpret_cast<volatile int*>(&r.idx[slot]);
    mbar_arrive(&r.empty[slot]);
    if (t < 0) return 0;
    T = decode_tile(a, t);
    return 1;
}

// Consumer, a whole warp (every lane waits and reads; lane 0 frees the slot for the warp).
__device__ __forceinline__ int tile_ring_get_warp(TileRing& r, uint32_t n, const AttnArgs& a, Tile& T,
                                                  volatile int* abort_flag, int lane) {
    const uint32_t slot = n % kTileRing;
    const bool w = __all_sync(0xFFFFFFFFu, mbar_wait(&r.full[slot], (n / kTileRing) & 1, abort_flag, a.err));
    if (!w) return -1;
    const int t = *reinterpret_cast<volatile int*>(&r.idx[slot]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&r.empty[slot]);
    if (t < 0) return 0;
    T = decode_tile(a, t);
    return 1;
}

}  // namespace bsa

