// Run-time work distribution for the persistent tensor-core kernels.
//
// Items are dealt out at run time rather than round-robin: the TMA warp of
// each CTA claims the next item index from a counter in the workspace
// (atomicAdd), so a CTA that runs faster (its SM closer to the data, or its
// items cheaper) simply takes more of them and all CTAs finish close
// together; the work table lists long examples first, so the last items
// claimed are the cheap ones. The claiming warp passes each item to the
// CTA's other roles through a small ring in shared memory guarded by
// mbarriers (one `full` arrival per posted item, one `empty` arrival per
// consumer warp). A posted item with head = -1 marks the end.
//
// Claims run two items ahead of the item being posted, so the counter's and
// the table's global-memory latency overlaps the current item's work (and
// the producer can prefetch the next item's tiles into L2).
#pragma once

#include "ba_common.cuh"
#include "ba_ptx.cuh"

namespace ba {

constexpr int kItemRing = 4;

// Counters (one per kernel of a call) sit in the workspace's status block,
// after the status word; the work-list kernel zeroes them.
constexpr int kCounterFwd = 32, kCounterDq = 33, kCounterDkdv = 34;

struct ItemRing {
    int4 item[kItemRing];  // {first row of the example, its length, tile, head}; head < 0: no more items
    int2 other[kItemRing]; // the other side's {first row, length} (cross-attention; else the same)
    uint64_t full[kItemRing], empty[kItemRing];
};

// One thread initialises the ring; `consumers` warps read every item.
__device__ __forceinline__ void item_ring_init(ItemRing &q, uint32_t consumers)
{
    for (int i = 0; i < kItemRing; ++i) {
        mbar_init(&q.full[i], 1);
        mbar_init(&q.empty[i], consumers);
    }
}

// The claiming side (all 32 lanes of the TMA warp call every member).
struct ItemSource {
    const int4 *table;
    const int32_t *other; // cross-attention: the other side's offsets, else nullptr
    int *counter;
    uint32_t total, heads;
    uint32_t next;     // claimed, not yet posted
    int4 next_info;    // its table entry
    int2 next_other{0, 0}; // its other side's rows (cross-attention)
    uint32_t pending;  // claimed after `next` (lane 0's atomic result)
    uint32_t posted = 0;

    __device__ __forceinline__ ItemSource(const int4 *t, int32_t entries, int32_t h, int *ctr,
                                          const int32_t *other_offsets = nullptr)
        : table(t), other(other_offsets), counter(ctr), total(uint32_t(entries) * uint32_t(h)), heads(uint32_t(h))
    {
        uint32_t a = 0, b = 0;
        if ((threadIdx.x & 31) == 0) {
            a = atomicAdd(reinterpret_cast<unsigned int *>(counter), 1u);
            b = atomicAdd(reinterpret_cast<unsigned int *>(counter), 1u);
        }
        next = __shfl_sync(0xffffffffu, a, 0);
        pending = b;
        load_next();
    }

    // next's table entry, and (cross-attention) its example's other side; for
    // self-attention nothing waits on the load here (its result is first used
    // at the next advance)
    __device__ __forceinline__ void load_next()
    {
        next_info = next < total ? table[next / heads] : make_int4(0, 0, 0, 0);
        if (other && next < total) {
            const int32_t o0 = other[next_info.w];
            next_other = make_int2(o0, other[next_info.w + 1] - o0);
        }
    }

    __device__ __forceinline__ void decode(uint32_t n, const int4 &info, const int2 &oth, TileRef &r) const
    {
        r.b = info.w;
        r.h = int32_t(n % heads);
        r.s0 = info.x;
        r.L = info.y;
        r.t = info.z;
        r.os0 = other ? oth.x : info.x;
        r.oL = other ? oth.y : info.y;
    }

    // The item after the one advance() returned last, if any (for L2 prefetches).
    __device__ __forceinline__ bool peek(TileRef &r) const
    {
        if (next >= total) return false;
        decode(next, next_info, next_other, r);
        return true;
    }

    // Posts the next item to the ring and returns it in r; at the end posts
    // the end marker and returns false. ok becomes false after a timed-out wait.
    __device__ __forceinline__ bool advance(TileRef &r, ItemRing &q, volatile int *abort, bool &ok)
    {
        const uint32_t slot = posted % kItemRing;
        if (!mbar_wait(&q.empty[slot], ((posted / kItemRing) & 1) ^ 1, abort)) {
            ok = false;
            return false;
        }
        const bool more = next < total;
        if (more) decode(next, next_info, next_other, r);
        if ((threadIdx.x & 31) == 0) {
            q.item[slot] = more ? make_int4(r.s0, r.L, r.t, r.h) : make_int4(0, 0, 0, -1);
            q.other[slot] = make_int2(r.os0, r.oL);
            mbar_arrive(&q.full[slot]);
        }
        __syncwarp();
        ++posted;
        if (!more) return false;
        // move the lookahead on: the pending claim becomes the next item, and one more is claimed
        next = __shfl_sync(0xffffffffu, pending, 0);
        load_next();
        if ((threadIdx.x & 31) == 0) pending = atomicAdd(reinterpret_cast<unsigned int *>(counter), 1u);
        return true;
    }
};

// The reading side (all 32 lanes of each consumer warp call advance()).
struct ItemSink {
    uint32_t taken = 0;

    // The next posted item into r; false at the end marker, or (with ok set
    // false) after a timed-out wait.
    __device__ __forceinline__ bool advance(TileRef &r, ItemRing &q, volatile int *abort, bool &ok)
    {
        const uint32_t slot = taken % kItemRing;
        if (!mbar_wait(&q.full[slot], (taken / kItemRing) & 1, abort)) {
            ok = false;
            return false;
        }
        const int4 it = q.item[slot];
        const int2 ot = q.other[slot];
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&q.empty[slot]);
        ++taken;
        if (it.w < 0) return false;
        r.b = -1; // not carried by the ring (no consumer of these kernels reads it)
        r.s0 = it.x;
        r.L = it.y;
        r.t = it.z;
        r.h = it.w;
        r.os0 = ot.x;
        r.oL = ot.y;
        return true;
    }
};

// Static dealing for kernels where the ring's extra code costs more than the
// balance gains (measured: the dK/dV pass, whose instruction footprint is at
// the edge of the instruction cache): CTA c takes items c, c + grid, ... in
// table order; each role walks the same sequence itself (same interface as
// ItemSink / ItemSource, ring unused).
struct StaticItems {
    const int4 *table;
    const int32_t *other;
    uint32_t total, heads, n;
    int4 next;
    __device__ __forceinline__ StaticItems(const int4 *t, int32_t entries, int32_t h, const int32_t *other_offsets)
        : table(t), other(other_offsets), total(uint32_t(entries) * uint32_t(h)), heads(uint32_t(h)), n(blockIdx.x),
          next()
    {
        if (n < total) next = table[n / heads];
    }
    __device__ __forceinline__ bool peek(TileRef &r) const
    {
        if (n >= total) return false;
        r.b = next.w;
        r.h = int32_t(n % heads);
        r.s0 = next.x;
        r.L = next.y;
        r.t = next.z;
        if (other) {
            r.os0 = other[next.w];
            r.oL = other[next.w + 1] - r.os0;
        } else {
            r.os0 = r.s0;
            r.oL = r.L;
        }
        return true;
    }
    __device__ __forceinline__ bool advance(TileRef &r, ItemRing &, volatile int *, bool &)
    {
        if (!peek(r)) return false;
        n += gridDim.x;
        if (n < total) next = table[n / heads];
        return true;
    }
};

} // namespace ba
