// schedule.cuh -- split-KV work distribution shared by the main and combine
// kernels (device side; computed from the lengths that live on the device, so
// a run needs no host synchronisation and can be captured in a CUDA graph).
//
// The KV tiles (kTileKV rows each) of all sequences are laid end to end:
// sequence b owns tiles [acc_b, acc_b + n_b) of a flat index space of N_t
// tiles.  The space is cut into P equal contiguous ranges of T = ceil(N_t/P)
// tiles ("partitions"); partition p is processed by one CTA (or CTA pair) per
// query-row group.  A sequence that falls inside one partition is finished by
// that CTA; a sequence cut by partition boundaries leaves one fp32 partial
// (O / l and its log-sum-exp) per piece, merged by the combine kernel.
//
// Partial slots: partition p owns slots 2p and 2p+1.  The piece of sequence b
// in partition p uses slot 2p if b started before p, else slot 2p+1 (b starts
// in p and continues after it).  Both can occur in one partition, for two
// different sequences; a sequence that both starts before and ends after p is
// p's only sequence and uses 2p.
//
// Batch-invariant schedule (S > 0 tiles).  Where a sequence is cut above
// depends on every other sequence of the batch, and so do the rounding of
// its partials and of their merge.  With S > 0 the unit of work is instead a
// chunk of S tiles of one sequence (its last chunk shorter): chunk k of
// sequence b covers tiles [kS, min(kS + S, n_b)), is always a piece of its
// own, and a sequence of u_b > 1 chunks writes chunk k to slot acc_b + k
// (acc_b = chunks of the sequences before b).  The flat list of chunks is cut
// into P equal ranges as before; only which CTA computes a chunk depends on
// the batch, not what it computes, so a sequence's output is bitwise the same
// in any batch.
#pragma once

#include <cstdint>

namespace mla {

constexpr int kTileKV = 128;       // kv rows per pipeline tile
constexpr int kDqk = 576;          // 512 latent + 64 rope
constexpr int kDv = 512;
constexpr int kChunk = 64;         // columns per 128-byte swizzled chunk
constexpr int kNumChunks = kDqk / kChunk;  // 9

// status word bits (workspace header, word 0)
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusSeqlen = 2u;

__device__ __forceinline__ int clamp_len(int L, int L_max, uint32_t* status) {
    if (L < 0 || L > L_max) {
        if (status) atomicOr(status, kStatusSeqlen);
        L = L < 0 ? 0 : L_max;
    }
    return L;
}

__device__ __forceinline__ int num_tiles(int L) { return (L + kTileKV - 1) / kTileKV; }

// schedule units of a sequence of L keys: its tiles (S = 0) or its S-tile chunks
__device__ __forceinline__ long long num_units(int L, int S) {
    const long long n = num_tiles(L);
    return S > 0 ? (n + S - 1) / S : n;
}

// Warp-cooperative: total tiles over all sequences, and (for `start`) the
// first sequence whose tiles reach past `start` with its flat offset.
// Every lane returns the same values.
struct ScanResult {
    long long total;     // N_t
    int b_first;         // first sequence with acc_b + n_b > start (or B)
    long long acc_first; // acc of b_first
};

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Schedule actually used for a run (warp-cooperative; every CTA and the
// combine kernel reach the same answer from the same lengths).  A plan's
// split_tiles > 0 (batch-invariant) is kept.  Otherwise the balanced schedule
// is used, except when a whole sequence per partition is expected to finish
// sooner: cutting a sequence costs about kCutTiles tiles of time (an extra
// epilogue that stalls the pipeline, the fp32 partials and their merge), and
// a balanced partition holds up to two cut pieces.  So when every non-empty
// sequence fits its own partition, the sequences keep at least half of the
// partitions busy, and the longest sequence is no longer than the balanced
// share plus two cuts, each sequence is one piece (returned as a chunk size
// covering the longest sequence).
constexpr long long kCutTiles = 5;

struct ScheduleScan {
    int S;             // chunk size in tiles of this run's schedule (0: balanced over tiles)
    long long units;   // schedule units over all sequences (tiles, or chunks)
    long long acc_at;  // units of the sequences before sequence `b_at` (0 when b_at < 0)
};

// One pass over the lengths (warp-cooperative): the schedule of this run, its
// number of units and, for b_at >= 0, the flat unit offset of sequence b_at.
// Every quantity whose unit depends on the schedule is accumulated for each
// candidate (tiles; chunks of the plan's size; non-empty sequences, the unit of
// the one-piece-per-sequence schedule), so one pass serves all three.
__device__ inline ScheduleScan schedule_scan_warp(const int32_t* seqlens, int B, int L_max, int P, int plan_split,
                                                  int b_at = -1) {
    const int lane = threadIdx.x & 31;
    long long total = 0, n_max = 0, nonempty = 0, chunks = 0;
    long long at_tiles = 0, at_nonempty = 0, at_chunks = 0;
    for (int b = lane; b < B; b += 32) {
        const int L = clamp_len(__ldg(seqlens + b), L_max, nullptr);
        const long long n = num_tiles(L);
        const long long c = plan_split > 0 ? num_units(L, plan_split) : 0;
        total += n;
        n_max = n > n_max ? n : n_max;
        nonempty += (n > 0);
        chunks += c;
        if (b < b_at) {
            at_tiles += n;
            at_nonempty += (n > 0);
            at_chunks += c;
        }
    }
    total = warp_sum_ll(total);
    nonempty = warp_sum_ll(nonempty);
    chunks = warp_sum_ll(chunks);
    at_tiles = warp_sum_ll(at_tiles);
    at_nonempty = warp_sum_ll(at_nonempty);
    at_chunks = warp_sum_ll(at_chunks);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const long long y = __shfl_xor_sync(0xffffffffu, n_max, o);
        n_max = y > n_max ? y : n_max;
    }
    if (plan_split > 0) return {plan_split, chunks, at_chunks};
    if (n_max == 0 || nonempty > P || 2 * nonempty < P) return {0, total, at_tiles};
    const long long T = (total + P - 1) / P;
    if (n_max <= T + 2 * kCutTiles) return {static_cast<int>(n_max), nonempty, at_nonempty};
    return {0, total, at_tiles};
}

// Locate the first sequence overlapping flat unit `start` (warp-cooperative).
__device__ inline void locate_warp(const int32_t* seqlens, int B, int L_max, int S, long long start, int* b_out,
                                   long long* acc_out) {
    const int lane = threadIdx.x & 31;
    long long acc = 0;
    for (int base = 0; base < B; base += 32) {
        const int b = base + lane;
        const long long n = (b < B) ? num_units(clamp_len(__ldg(seqlens + b), L_max, nullptr), S) : 0;
        // inclusive prefix within the warp
        long long incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const long long excl = incl - n;
        // sequences with n > 0 whose range [acc+excl, acc+incl) reaches past start
        const bool hit = (b < B) && (n > 0) && (acc + incl > start);
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            const long long e = __shfl_sync(0xffffffffu, excl, src);
            *b_out = base + src;
            *acc_out = acc + e;
            return;
        }
        acc += __shfl_sync(0xffffffffu, incl, 31);
    }
    *b_out = B;
    *acc_out = acc;
}

struct Piece {
    int b;          // sequence
    int L;          // its (clamped) length
    int tile_lo;    // first tile (sequence-local index)
    int tile_hi;    // one past the last tile
    int slot;       // partial slot, or -1 when the piece is the whole sequence
};

// Sequential walker over the pieces of one partition; every role of a CTA
// runs its own copy and sees the same sequence of pieces.
struct PieceWalker {
    const int32_t* seqlens;
    int B, L_max, p;
    int S;                 // 0: balanced schedule over tiles; > 0: chunks of S tiles
    long long start, end;  // flat unit range of this partition
    int b;                 // next sequence to look at
    long long acc;         // its flat offset (in units)
    long long k;           // S > 0: next chunk of sequence b

    __device__ bool next(Piece& out) {
        if (S > 0) return next_chunk(out);
        while (b < B && acc < end) {
            const int L = clamp_len(__ldg(seqlens + b), L_max, nullptr);
            const long long n = num_tiles(L);
            const long long lo = acc > start ? acc : start;
            const long long hi = (acc + n) < end ? (acc + n) : end;
            const int cur = b;
            const long long acc_cur = acc;
            ++b;
            acc += n;
            if (hi <= lo) continue;
            out.b = cur;
            out.L = L;
            out.tile_lo = static_cast<int>(lo - acc_cur);
            out.tile_hi = static_cast<int>(hi - acc_cur);
            const bool starts_before = acc_cur < start;
            const bool continues_after = acc_cur + n > end;
            if (!starts_before && !continues_after) out.slot = -1;
            else out.slot = starts_before ? 2 * p : 2 * p + 1;
            return true;
        }
        return false;
    }

    // batch-invariant schedule: one S-tile chunk per piece
    __device__ bool next_chunk(Piece& out) {
        while (b < B && acc + k < end) {
            const int L = clamp_len(__ldg(seqlens + b), L_max, nullptr);
            const long long n = num_tiles(L);
            const long long u = (n + S - 1) / S;
            if (acc + k < start) k = start - acc;
            if (k >= u) {
                acc += u;
                ++b;
                k = 0;
                continue;
            }
            out.b = b;
            out.L = L;
            out.tile_lo = static_cast<int>(k * S);
            out.tile_hi = static_cast<int>((k + 1) * S < n ? (k + 1) * S : n);
            out.slot = (u == 1) ? -1 : static_cast<int>(acc + k);
            ++k;
            return true;
        }
        return false;
    }
};

}  // namespace mla
