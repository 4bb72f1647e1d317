// Tensor-core index scan for sm_100a ("FlashMemory-DeepSeek-V4 ... Lookahead
// Sparse Attention", gist.science technical summary, section 2.1 "Scoring
// Mechanism"):  z_s = sum_j w_j ReLU(q_j . k_s) for every entry s.
//
// Per sequence the q.k block is a dense contraction [entries x d] x [d x H]
// (H = 64 heads, d = 128: 16 Kflop per entry), so the scan is HBM-bound only
// when the dot products run on the tensor cores.  One kernel, persistent CTAs
// (one per SM), each streaming a contiguous range of tiles (128 entries for
// bf16 keys, 256 for e4m3 keys; tiles never straddle two sequences):
//   * warp 0 (producer): TMA loads of key tiles (128-byte swizzle) into a smem
//     ring -- the first ring's worth before anything else -- and, on every
//     sequence change from the third sequence on, builds that sequence's query
//     operand and gate weights in one of two smem slots (the first two are
//     built by the epilogue warps while the first keys load; no separate
//     preparation kernel);
//   * warp 1: tcgen05.mma, M = 128 entries per instruction, into a ring of
//     TMEM accumulators.  bf16 keys: N = H heads, the MMAs of two tiles issued
//     interleaved.  e4m3 keys: N = 2H (both query pieces side by side), the
//     two 128-entry halves of a tile issued interleaved.  Here an MMA costs the
//     tensor pipe about 50 cycles whatever its N (32 to 128), so the layout
//     keeps MMAs per byte low: 8 per 32 KB of keys in both cases (putting the
//     e4m3 pieces along K instead doubles them, and the MMAs then pace the
//     scan);
//   * warps 2-9: two epilogue warpgroups taking alternate tiles (a warpgroup's
//     per-tile chain of barrier wait, TMEM loads and arithmetic paced the scan
//     when both worked on every tile), one TMEM lane (= one entry) per thread:
//     the two pieces' products added (e4m3), ReLU, gate weights, head sum in
//     registers, one coalesced fp32 store per entry; the row scale comes from
//     shared memory.
// bf16 keys use kind::f16 (bf16 x bf16).  e4m3 keys use kind::f8f6f4 against
// an exact two-piece e4m3 split of the bf16 query, so the keys go from HBM to
// the tensor core untouched; the per-row key scale and the per-head
// power-of-two query scale are applied after the ReLU, which is positively
// homogeneous.
//
// The listed variant scores only the entries of a per-sequence index list (the
// kept set, re-ranked every decode step): the producer warp gathers those key
// rows with cp.async into the same swizzled layout, three tiles in flight per
// lane.
//
// A query slot is rewritten only after the MMA and all eight epilogue warps
// have released the sequence that used it (release barriers indexed by the
// sequence's ordinal mod 8, so a warp running ahead never completes an older
// phase).  Every wait is bounded in time; a wait that gives up sets
// LSA_ERR_TIMEOUT in the caller's error word, stops the CTA's loops, drains the
// issued MMAs and frees TMEM before returning.
#include <cuda.h>

#include "lsa_internal.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace ptx;

enum Kind { BF16_D128 = 0, BF16_D64 = 1, E4M3_D128 = 2, E4M3_D64 = 3 };

__host__ __device__ constexpr bool is_e4m3(int kind) { return kind == E4M3_D128 || kind == E4M3_D64; }

template <int KIND>
struct Cfg;
// Per key type: a tile is kSub sub-tiles of 128 rows (one MMA row block each);
// a stage holds one tile, loaded as kBoxes TMA boxes of 128 bytes x kBoxRows
// rows; the query operand has H rows (N of the MMA), of d elements (bf16) or
// two e4m3 pieces of d elements each, piece 2's rows after piece 1's (e4m3).
template <>
struct Cfg<BF16_D128> {
    static constexpr int kSub = 1;
    static constexpr int kStageBytes = 32768;   // 128 rows x 128 bf16
    static constexpr int kBoxes = 2;            // two 64-element (128-byte) column boxes
    static constexpr int kBoxRows = 128;
    static constexpr int kQBytesPerHead = 256;
    static constexpr int kStages = 5;
};
template <>
struct Cfg<BF16_D64> {
    static constexpr int kSub = 1;
    static constexpr int kStageBytes = 16384;
    static constexpr int kBoxes = 1;
    static constexpr int kBoxRows = 128;
    static constexpr int kQBytesPerHead = 128;
    static constexpr int kStages = 8;
};
template <>
struct Cfg<E4M3_D128> {
    static constexpr int kSub = 2;              // 256-row tiles: half as many tile steps per byte
    static constexpr int kStageBytes = 32768;   // 256 rows x 128 e4m3
    static constexpr int kBoxes = 1;
    static constexpr int kBoxRows = 256;
    static constexpr int kQBytesPerHead = 256;  // two e4m3 pieces x 128
    static constexpr int kStages = 5;           // 160 KB of keys in flight per SM, as for bf16 keys
};
// e4m3 keys with d = 64: 64-byte rows in the 64-byte-swizzled K-major layout (the
// 128-byte swizzle needs 128-byte rows); 256-row tiles of 16 KB, each sub-tile
// two K = 32 MMAs, so again 8 MMAs per 32 KB of keys; twice the stages of the
// d = 128 ring for the same bytes in flight.
template <>
struct Cfg<E4M3_D64> {
    static constexpr int kSub = 2;
    static constexpr int kStageBytes = 16384;   // 256 rows x 64 e4m3
    static constexpr int kBoxes = 1;
    static constexpr int kBoxRows = 256;
    static constexpr int kQBytesPerHead = 128;  // two e4m3 pieces x 64
    static constexpr int kStages = 10;          // 160 KB of keys in flight per SM, as for bf16 keys
};

// Key row bytes, and where 16-byte chunk c of row r of a stage sits: the TMA
// writes a stage in this layout and the MMA descriptors read it.  128-byte rows
// use the 128-byte swizzle (bf16 d = 128 keys are two such column boxes, 16 KB
// apart); 64-byte rows the 64-byte swizzle.
template <int KIND>
__host__ __device__ constexpr int row_bytes() {
    return KIND == BF16_D128 ? 256 : KIND == E4M3_D64 ? 64 : 128;
}
template <int KIND>
__device__ __forceinline__ uint32_t stage_chunk_off(int r, int c) {
    if (KIND == E4M3_D64) return uint32_t(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
    return uint32_t((c >> 3) * 16384 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}
template <int KIND>
__device__ __forceinline__ uint64_t kdesc(uint32_t addr) {
    return KIND == E4M3_D64 ? desc_sw64(addr) : desc_sw128(addr);
}

constexpr int kThreads = 320;         // warp 0 producer, warp 1 MMA, warps 2-9 epilogue (2 warpgroups)
constexpr int kEpiGroups = 2;
constexpr int kEpiWarps = 8;
constexpr int kRel = 8;               // query-slot release barriers, by sequence ordinal mod kRel
constexpr int kRows = 128;            // rows of one MMA (M) and of a sub-tile
constexpr int kAccMax = 8;            // TMEM accumulator stages at most
constexpr int kScaleSlotsMax = 24;    // row-scale ring slots at most (stages + accumulators)
constexpr int kDoneMax = 24;          // tile-completion barriers at most (per accumulator + per stage)
constexpr int kMaxB = 512;            // sequences per launch on this path
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per wait

template <int KIND>
__host__ __device__ constexpr int tile_rows() {
    return kRows * Cfg<KIND>::kSub;
}
// TMEM columns of one sub-tile's accumulator (fp32, one per head and query
// piece: e4m3 keys give columns [0, H) for piece 1 and [H, 2H) for piece 2,
// added by the epilogue before the ReLU) and of one tile's.
template <int KIND, int H>
__host__ __device__ constexpr int sub_cols() {
    return is_e4m3(KIND) ? 2 * H : H;
}
template <int KIND, int H>
__host__ __device__ constexpr int tile_cols() {
    return sub_cols<KIND, H>() * Cfg<KIND>::kSub;
}
// Tile accumulators held in TMEM (512 columns per SM).
template <int KIND, int H>
__host__ __device__ constexpr int acc_tiles() {
    return 512 / tile_cols<KIND, H>() < kAccMax ? 512 / tile_cols<KIND, H>() : kAccMax;
}
// Tiles whose MMAs are issued together, interleaved so that consecutive MMAs
// write different accumulators: a chain of MMAs into one accumulator waits on
// each accumulation, independent chains overlap in the tensor pipe.  The two
// halves of a 256-row tile already give two chains.
template <int KIND, int H>
__host__ __device__ constexpr int mma_group() {
    return Cfg<KIND>::kSub == 2 ? 1 : 2;
}
__host__ __device__ constexpr uint32_t tmem_cols(int cols) {
    return cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : cols <= 256 ? 256 : 512;
}

template <int KIND, int H>
__host__ __device__ constexpr int qimg_bytes() {
    return Cfg<KIND>::kQBytesPerHead * H;
}

// cp.async of 16 bytes (zero-filled when src_bytes == 0).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// 4-byte cp.async (zero-filled when src_bytes == 0).
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// Arrive on `bar` once every cp.async this thread has issued so far has completed (the barrier's
// expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Query operand of one sequence, built by nw warps (the 8 epilogue warps at
// kernel start, the producer warp later) straight into a shared-memory slot,
// laid out exactly as the MMA reads it
// (K-major, 128-byte swizzle: 16-byte chunk c of row j at chunk c ^ (j % 8)),
// plus the gate weights w' the epilogue applies.
//
// bf16 keys: the bf16 query itself, w' = w.
// e4m3 keys: per head j, a power-of-two scale 2^e_j brings max_c |q_jc| into
// [128, 256); p1 = e4m3(q 2^e_j), p2 = e4m3(q 2^e_j - p1), both round to
// nearest even.  A bf16 value has 8 significant bits, p1 carries 4 and the
// remainder q 2^e_j - p1 is a multiple of the bf16 ulp no larger than 8 ulps,
// so p2 holds it exactly whenever it is at least the e4m3 subnormal step 2^-9:
// p1 + p2 == q 2^e_j for every element with |q| >= 2^-10 max_c |q_jc|, and
// within 2^-10 of it (2^-17 max_c |q_jc| before scaling) otherwise.  The two
// pieces are rows [0, H) and [H, 2H) of one operand.  w'_j = w_j 2^-e_j.
// ---------------------------------------------------------------------------
// 2^e as a float, for -126 <= e <= 127.
__device__ __forceinline__ float pow2f(int e) { return __int_as_float(uint32_t(e + 127) << 23); }
// v * 2^e with a single rounding (like ldexpf), for -126 <= e <= 254.
__device__ __forceinline__ float scale_pow2(float v, int e) {
    if (e > 127) {   // exact: v * 2^127 stays finite because |v| < 2^(8 - e) here
        v *= pow2f(127);
        e -= 127;
    }
    return v * pow2f(e);
}
// The exponent E of m > 0 in the frexp sense: m = f * 2^E with 0.5 <= f < 1.
__device__ __forceinline__ int frexp_exponent(float m) {
    const uint32_t bits = __float_as_uint(m);
    const int ex = int(bits >> 23);
    return ex ? ex - 126 : (32 - __clz(int(bits & 0x7FFFFFu))) - 149;
}

template <int KIND, int H>
__device__ __forceinline__ void build_query(const uint16_t *__restrict__ qb, const float *__restrict__ wb, int d,
                                            uint8_t *slot, float *wsm, int wi, int nw, int lane) {
    if (!is_e4m3(KIND)) {
        // 16-byte chunks, all of a thread's loads in flight before its stores
        const int cpr = d / 8;
        const int tid = wi * 32 + lane, nthr = nw * 32;
        const uint32_t s_u32 = smem_u32(slot);
        for (int i0 = 0; i0 < H * cpr; i0 += nthr * 16) {
            uint4 v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int i = i0 + u * nthr + tid;
                if (i < H * cpr) {
                    const int j = i / cpr, c = i % cpr;
                    v[u] = *reinterpret_cast<const uint4 *>(qb + j * d + c * 8);
                }
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int i = i0 + u * nthr + tid;
                if (i < H * cpr) {
                    const int j = i / cpr, c = i % cpr;
                    const uint32_t dst = s_u32 + (c >> 3) * (H * 128) + j * 128 + (((c & 7) ^ (j & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[u].x), "r"(v[u].y),
                                 "r"(v[u].z), "r"(v[u].w)
                                 : "memory");
                }
            }
        }
        for (int j = wi * 32 + lane; j < H; j += nw * 32) wsm[j] = wb[j];
    } else {
        // d / 16 threads per head (8 for d = 128, 4 for d = 64), thread g of a head owns channels
        // 16g .. 16g+15 (one 16-byte chunk of each piece): the head's max is a 3- or 2-step shuffle and
        // each thread converts 16 channels.  Two heads per thread per iteration, both heads' loads issued
        // before any arithmetic (one global round trip for the 8-warp build of 64 heads)
        constexpr int DK = KIND == E4M3_D64 ? 64 : 128;
        constexpr int TPH = DK / 16;   // threads per head
        constexpr int LOG_TPH = TPH == 8 ? 3 : 2;
        const int tid = wi * 32 + lane, nthr = nw * 32;
        const int g = tid & (TPH - 1);
        const int hstride = nthr >> LOG_TPH;   // heads per round
        // every lane of a warp takes the same trip count (32 / TPH heads per warp, H a multiple of 16)
        for (int j0 = tid >> LOG_TPH; j0 < H; j0 += 2 * hstride) {
            uint4 ra[2], rb[2];
            float wj[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = j0 + h * hstride;
                if (j < H) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(qb + j * DK + 16 * g);
                    ra[h] = src[0];
                    rb[h] = src[1];
                    wj[h] = wb[j];
                } else {
                    ra[h] = rb[h] = make_uint4(0u, 0u, 0u, 0u);
                    wj[h] = 0.f;
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = j0 + h * hstride;   // uniform across the TPH threads of a head
                const uint32_t wds[8] = {ra[h].x, ra[h].y, ra[h].z, ra[h].w, rb[h].x, rb[h].y, rb[h].z, rb[h].w};
                float v[16];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    v[2 * c] = __uint_as_float(wds[c] << 16);
                    v[2 * c + 1] = __uint_as_float(wds[c] & 0xFFFF0000u);
                }
                float m = 0.f;
#pragma unroll
                for (int c = 0; c < 16; ++c) m = fmaxf(m, fabsf(v[c]));
#pragma unroll
                for (int o = TPH / 2; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                const int e = m > 0.f ? 8 - frexp_exponent(m) : 0;   // m 2^e in [128, 256)
                uint32_t p1w[4] = {0u, 0u, 0u, 0u}, p2w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int c = 0; c < 16; c += 2) {   // two channels per conversion (.x -> low byte)
                    const float2 sv = make_float2(scale_pow2(v[c], e), scale_pow2(v[c + 1], e));
                    const __nv_fp8x2_storage_t p1 = __nv_cvt_float2_to_fp8x2(sv, __NV_SATFINITE, __NV_E4M3);
                    const float2 h1 = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(p1, __NV_E4M3)));
                    const __nv_fp8x2_storage_t p2 =
                        __nv_cvt_float2_to_fp8x2(make_float2(sv.x - h1.x, sv.y - h1.y), __NV_SATFINITE, __NV_E4M3);
                    p1w[c >> 2] |= uint32_t(p1) << (8 * (c & 3));
                    p2w[c >> 2] |= uint32_t(p2) << (8 * (c & 3));
                }
                if (j < H) {
                    // the query operand in the keys' layout: row j (piece 1) and row H + j (piece 2); H is a
                    // multiple of 8, so both rows have the same swizzle phase
                    const int off =
                        DK == 128 ? j * 128 + ((g ^ (j & 7)) << 4) : j * 64 + ((g ^ ((j >> 1) & 3)) << 4);
                    *reinterpret_cast<uint4 *>(slot + off) = make_uint4(p1w[0], p1w[1], p1w[2], p1w[3]);
                    *reinterpret_cast<uint4 *>(slot + H * DK + off) = make_uint4(p2w[0], p2w[1], p2w[2], p2w[3]);
                    if (g == 0) wsm[j] = ldexpf(wj[h], -e);
                }
            }
        }
    }
}

// Whether the row scales of a tile (rows row0 .. row0+nvalid-1) travel by one bulk copy: the aligned
// superset [row0 & ~3, (row0 + nvalid + 3) & ~3) of 16-byte-aligned scales inside the array's scale_len
// entries.  Otherwise the producer copies them 4 bytes at a time.
__device__ __forceinline__ bool scales_bulk(int64_t row0, int64_t nvalid, int64_t scale_len, const float *k_scale) {
    return (reinterpret_cast<uintptr_t>(k_scale) & 15) == 0 && ((row0 + nvalid + 3) & ~int64_t(3)) <= scale_len;
}

// Sequence and rows of tile t; `b` is a cursor that only moves forward.
template <int TR>
__device__ __forceinline__ void tile_info(const int64_t *s_toff, const int64_t *s_seq, int B, int64_t t, int &b,
                                          int64_t &row0, int64_t &row_end) {
    while (b < B - 1 && t >= s_toff[b + 1]) ++b;
    row0 = s_seq[b] + (t - s_toff[b]) * TR;
    row_end = s_seq[b + 1];
}

// LISTED = false: every entry of every sequence (key tiles by TMA).
// LISTED = true:  entries idx[idx_off[b] ..] of each sequence (rows gathered
//                 by the producer warp with cp.async); z is written at the list
//                 position.
// SEL (full mode only): the selection's ballots fused into the epilogue (sel_bits, sel_cnt).
template <int KIND, int H, bool LISTED, bool SEL = false>
__global__ void __launch_bounds__(kThreads, 1)
scan_tc(const __grid_constant__ CUtensorMap tmap, const uint8_t *__restrict__ kbytes,
        const uint16_t *__restrict__ q, const float *__restrict__ w, int d, const int64_t *__restrict__ seq_off,
        const int32_t *__restrict__ idx, const int64_t *__restrict__ idx_off, int64_t list_cap, int B,
        const float *__restrict__ k_scale, int64_t scale_len, int64_t axis_cap, float *__restrict__ z,
        float *__restrict__ I, uint32_t *__restrict__ sel_bits, int32_t *__restrict__ sel_cnt, int32_t *err) {
    using C = Cfg<KIND>;
    constexpr int S = C::kStages;
    constexpr int QIMG = qimg_bytes<KIND, H>();
    constexpr int TR = tile_rows<KIND>();          // rows per tile
    constexpr int SUBC = sub_cols<KIND, H>();      // accumulator columns per 128-row sub-tile (MMA N)
    constexpr int TILEC = tile_cols<KIND, H>();    // accumulator columns per tile
    constexpr int KACC = acc_tiles<KIND, H>();     // tile accumulators
    constexpr int G = mma_group<KIND, H>();
    constexpr uint32_t NCOL = tmem_cols(KACC * TILEC);
    static_assert(G >= 1 && G <= KACC / 2, "the epilogue must own accumulators while a group is issued");
    static_assert(S >= G, "a group waits for G filled stages");
    // The epilogue warpgroups take alternate tiles (each warp has two tile times for one tile: a
    // warpgroup's wait / TMEM load / arithmetic chain per tile paced the kernel when both warpgroups
    // worked on every tile).  The MMA commits each tile's completion to a barrier per accumulator
    // (the epilogue waits there: the next phase is the tile KACC later, whose MMA needs this tile's
    // release by the waiting warpgroup itself).  A parity wait is only unambiguous while the barrier
    // cannot complete a second phase past the one waited for: the producer's wait for tile j - S may
    // share that barrier when S <= KACC (its next phase, tile j - S + KACC >= j, needs the producer's
    // own load of tile j); with more stages than accumulators tile j - S + KACC could complete before a
    // slow producer polls, so the MMA also commits to a barrier per stage, whose next phase is again
    // the producer's own load.
    constexpr bool kStageDone = S > KACC;
    static_assert(KACC + (kStageDone ? S : 0) <= kDoneMax, "completion barriers");
    // e4m3 keys: the per-row scales of each tile go to a shared-memory ring by cp.async (the
    // producer warp), never through a register load of an epilogue warp, whose wait on its TMEM
    // loads would otherwise also wait for that HBM load.  Slot j % RS holds tile j's scales; it is
    // rewritten for tile j + RS only after the MMA of tile j + KACC, i.e. after the epilogue of tile
    // j released its accumulator, which it does after reading the scales.
    constexpr bool kScales = is_e4m3(KIND);
    constexpr int RS = S + KACC;
    // a scale slot holds a tile's row scales from an aligned start: up to 3 leading and 4 trailing extra
    constexpr int SS = TR + 8;
    static_assert(!kScales || RS <= kScaleSlotsMax, "row-scale ring");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = smem;
    uint8_t *qimg = stages + S * C::kStageBytes;                  // 2 query slots
    uint64_t *full = reinterpret_cast<uint64_t *>(qimg + 2 * QIMG);  // [S] stage loaded
    uint64_t *qfull = full + S;                                   // [2] query slot built
    uint64_t *qrel = qfull + 2;                                   // [kRel] by sequence ordinal
    // the MMAs of a tile completed: [KACC] its accumulator is ready (and, with S <= KACC, its stage
    // free); then, with S > KACC, [S] its stage is free
    uint64_t *tdone = qrel + kRel;
    uint64_t *tfree = tdone + KACC;
    uint64_t *tempty = tdone + kDoneMax;                          // [KACC] accumulator read by the epilogue
    uint64_t *drain = tempty + kAccMax;
    uint64_t *sfull = drain + 1;                                  // [RS] row scales of a tile landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sfull + kScaleSlotsMax);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    int *s_nord = abort_flag + 1;                                 // sequences (ordinals) in this CTA's range
    // gate weights of the two slots, read as float4: 16-byte aligned
    float *wsm = reinterpret_cast<float *>((reinterpret_cast<uintptr_t>(tmem_slot + 4) + 15) & ~uintptr_t(15));
    int64_t *s_seq = reinterpret_cast<int64_t *>(wsm + 2 * H);   // [B+1] tile-axis offsets
    int64_t *s_toff = s_seq + (B + 1);                           // [B+1] first tile of each sequence
    int64_t *s_base = s_toff + (B + 1);                          // [B+1] entry base (listed mode)
    float *s_scale = reinterpret_cast<float *>((reinterpret_cast<uintptr_t>(s_base + (B + 1)) + 15) & ~uintptr_t(15));
    __shared__ int64_t s_range[2];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_v = abort_flag;

    // tile axis: the entries (full mode) or the list positions (listed mode); all offsets are
    // loaded at once, the tile prefix is then summed from shared memory.  Full mode over an axis an earlier
    // kernel produced (axis_cap > 0: the rows of a compacted key array, their offsets clamped to its
    // capacity) waits for that kernel first, like the listed mode
    {
        if (LISTED || axis_cap > 0) pdl_wait();
        const int64_t *axis = LISTED ? idx_off : seq_off;
        const int64_t acap = LISTED ? list_cap : axis_cap;
        for (int b = threadIdx.x; b <= B; b += kThreads) {
            int64_t a = axis[b];
            if (acap > 0 && a > acap) a = acap;
            s_seq[b] = a;
            s_base[b] = seq_off[b];
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int b = 0; b <= B; ++b) {
            s_toff[b] = acc;
            if (b < B) {
                const int64_t a = s_seq[b], a1 = s_seq[b + 1];
                acc += (a1 > a ? a1 - a + TR - 1 : 0) / TR;
            }
        }
        const int64_t T = acc;
        const int64_t t0 = T * blockIdx.x / gridDim.x, t1 = T * (blockIdx.x + 1) / gridDim.x;
        s_range[0] = t0;
        s_range[1] = t1;
        int nord = 0;   // sequences that own tiles in [t0, t1)
        for (int b = 0; b < B; ++b)
            if (s_toff[b + 1] > s_toff[b] && s_toff[b + 1] > t0 && s_toff[b] < t1) ++nord;
        *s_nord = nord;
        *abort_flag = 0;
        for (int s = 0; s < S; ++s) mbar_init(&full[s], LISTED ? 32 : 1);
        for (int s = 0; s < 2; ++s) mbar_init(&qfull[s], 1);
        for (int s = 0; s < kRel; ++s) mbar_init(&qrel[s], 1 + kEpiWarps);
        // an accumulator is released by the warps that read it: one warpgroup per 128-row sub-tile
        for (int s = 0; s < KACC; ++s) mbar_init(&tdone[s], 1);
        if (kStageDone)
            for (int s = 0; s < S; ++s) mbar_init(&tfree[s], 1);
        // an accumulator is released by the four warps of the warpgroup that read it
        for (int s = 0; s < KACC; ++s) mbar_init(&tempty[s], 4);
        mbar_init(drain, 1);
        // full mode: one arrival (the bulk copy's expect_tx, or lane 0 after the copies landed); listed
        // mode: one cp.async-tracked arrival per producer lane
        if (kScales)
            for (int s = 0; s < RS; ++s) mbar_init(&sfull[s], LISTED ? 32 : 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&tmap);
    if (warp == 1) {
        tmem_alloc(tmem_slot, NCOL);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int64_t t0 = s_range[0], t1 = s_range[1];
    const int nord = *s_nord;
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // builds the query operand of a new sequence (ordinal o) into slot o & 1
        // local tile j may be loaded once the MMA of tile j - S (same stage) has completed
        // completion barrier and parity of local tile i
        auto done_bar = [&](int64_t i) -> uint64_t * { return kStageDone ? &tfree[int(i % S)] : &tdone[int(i % KACC)]; };
        auto done_par = [&](int64_t i) -> uint32_t { return uint32_t((i / (kStageDone ? S : KACC)) & 1); };
        auto stage_free_test = [&](int64_t j) -> bool {
            return j < S || mbar_test_wait(done_bar(j - S), done_par(j - S));
        };
        auto stage_free_wait = [&](int64_t j) -> bool {
            return j < S || mbar_wait(done_bar(j - S), done_par(j - S), abort_v, kWaitLimitNs);
        };
        // row scales of local tile j (rows [row0, row_end) of the entry axis), all 32 lanes.  A span
        // that starts 16-byte aligned and has a multiple of 4 rows goes by one bulk copy (the copy
        // engine, like the keys); any other by 4-byte cp.async.  Global loads through the SM's L1 path
        // held the tensor pipe back by a factor of about four here, so the bulk path is the rule: it
        // takes every tile when the sequence offsets are multiples of 4.
        auto load_scales = [&](int64_t j, int64_t row0, int64_t row_end) {
            if (!kScales) return;
            const int slot = int(j % RS);
            const int64_t nvalid = (row_end - row0) < TR ? (row_end - row0) : TR;
            const int64_t a0 = row0 & ~int64_t(3), a1 = (row0 + nvalid + 3) & ~int64_t(3);
            if (scales_bulk(row0, nvalid, scale_len, k_scale)) {
                if (lane == 0) {   // the barrier's only arrival (no per-lane arrivals next to the MMA's reads)
                    mbar_arrive_expect_tx(&sfull[slot], uint32_t((a1 - a0) * 4));
                    bulk_load(s_scale + slot * SS, k_scale + a0, uint32_t((a1 - a0) * 4), &sfull[slot]);
                }
                return;
            }
            const uint32_t dst = smem_u32(s_scale + slot * SS);
#pragma unroll
            for (int k = 0; k < TR / 32; ++k) {
                const int r = lane + 32 * k;
                const bool valid = row0 + r < row_end;
                cp_async_4(dst + r * 4, k_scale + (valid ? row0 + r : 0), valid ? 4u : 0u);
            }
            cp_async_wait_all();   // unaligned spans only: the copies land, then one arrival
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfull[slot]);
        };
        // (ordinals 0 and 1 are built by the epilogue warps, idle at kernel start)
        auto next_query = [&](int b, int o) -> bool {
            if (o < 2) return true;
            bool ok = true;
            if (o >= 2)   // slot o & 1 last served ordinal o - 2: wait until every reader released it
                ok = mbar_wait(&qrel[(o - 2) % kRel], uint32_t(((o - 2) / kRel) & 1), abort_v, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) return false;
            build_query<KIND, H>(q + size_t(b) * H * d, w + size_t(b) * H, d, qimg + (o & 1) * QIMG,
                                 wsm + (o & 1) * H, 0, 1, lane);
            fence_proxy_async_smem();   // generic-proxy smem writes -> tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&qfull[o & 1]);
            return true;
        };
        if (!LISTED) {
            // the keys do not depend on the preceding kernel: fill the ring first
            const int64_t npre = (t1 - t0) < S ? (t1 - t0) : S;
            {
                int bp = 0;
                int64_t r0, r1;
                for (int64_t t = t0; t < t0 + npre; ++t) {
                    tile_info<TR>(s_toff, s_seq, B, t, bp, r0, r1);
                    const int st = int(t - t0);
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[st], C::kStageBytes);
#pragma unroll
                        for (int bx = 0; bx < C::kBoxes; ++bx)
                            tma_load_2d(stages + st * C::kStageBytes + bx * 16384, &tmap, &full[st], bx * 64,
                                        int(r0));
                    }
                    load_scales(t - t0, r0, r1);
                }
            }
            pdl_wait();
            int b = 0, cur = -1, qn = 0, st = 0;
            uint32_t ph = 0;
            int64_t row0, row_end;
            for (int64_t t = t0; t < t1; ++t) {
                tile_info<TR>(s_toff, s_seq, B, t, b, row0, row_end);
                if (b != cur) {
                    if (!next_query(b, qn)) break;
                    cur = b;
                    ++qn;
                }
                bool ok = true;
                if (t - t0 >= npre) {   // the first npre tiles were issued above
                    if (lane == 0) {
                        ok = stage_free_wait(t - t0);
                        if (ok) {
                            mbar_arrive_expect_tx(&full[st], C::kStageBytes);
#pragma unroll
                            for (int bx = 0; bx < C::kBoxes; ++bx)
                                tma_load_2d(stages + st * C::kStageBytes + bx * 16384, &tmap, &full[st], bx * 64,
                                            int(row0));
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (ok) load_scales(t - t0, row0, row_end);
                }
                if (!ok) break;
                if (++st == S) { st = 0; ph ^= 1; }
            }
        } else {
            // all 32 lanes gather: lane owns rows lane, lane + 32, ... of each tile; a stage (and its row
            // scales) is signalled by cp.async-tracked arrivals, one per lane
            pdl_wait();
            constexpr int RB = row_bytes<KIND>();
            constexpr int CPR = RB / 16;
            int b = 0, cur = -1, qn = 0, st = 0;
            uint32_t ph = 0;
            int64_t row0, row_end;
            for (int64_t t = t0; t < t1; ++t) {
                tile_info<TR>(s_toff, s_seq, B, t, b, row0, row_end);
                if (b != cur) {
                    if (!next_query(b, qn)) break;
                    cur = b;
                    ++qn;
                }
                const bool ok = stage_free_wait(t - t0);
                if (!__all_sync(0xffffffffu, ok)) break;
                const uint32_t stage_u32 = smem_u32(stages + st * C::kStageBytes);
#pragma unroll
                for (int rr = 0; rr < TR / 32; ++rr) {
                    const int r = lane + 32 * rr;
                    const int64_t p = row0 + r;
                    const bool valid = p < row_end;
                    const int64_t e = valid ? s_base[b] + idx[p] : 0;
                    const uint8_t *src = kbytes + e * RB;
#pragma unroll
                    for (int c = 0; c < CPR; ++c)
                        cp_async_16(stage_u32 + stage_chunk_off<KIND>(r, c), src + c * 16, valid ? 16u : 0u);
                    if (kScales)
                        cp_async_4(smem_u32(s_scale + int((t - t0) % RS) * SS + r), k_scale + e, valid ? 4u : 0u);
                }
                // each lane's arrival fires when its copies so far have landed: the stage is signalled as
                // soon as its own rows are in, while the next tile's gathers are already being issued
                cp_async_arrive_noinc(&full[st]);
                if (kScales) cp_async_arrive_noinc(&sfull[int((t - t0) % RS)]);
                if (++st == S) { st = 0; ph ^= 1; }
            }
            cp_async_wait_all();   // no copy into this CTA's shared memory outlives the loop
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = is_e4m3(KIND) ? idesc_e4m3(kRows, SUBC) : idesc_bf16(kRows, SUBC);
            // descriptors of stage 0 and slot 0; the others differ only in the start address field
            // (16-byte units), advanced incrementally: this thread's per-tile work is the tensor pipe's idle time
            const uint64_t a_desc0 = kdesc<KIND>(smem_u32(stages));
            const uint64_t b_desc0 = kdesc<KIND>(smem_u32(qimg));
            constexpr uint64_t kStageStep = uint64_t(C::kStageBytes >> 4);
            int b = 0, qn = -1, st = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            int64_t row0, row_end, seq_end = t0;   // seq_end: first tile of the next sequence
            uint64_t a_cur = a_desc0, b_cur = b_desc0;
            bool issued = false, ok = true;
            // A group of up to G tiles never continues past a sequence change: the query of a new
            // sequence is waited for only at the start of a group, once every earlier release is committed.
            for (int64_t t = t0; t < t1;) {
                if (t == seq_end) {   // first tile of a sequence (ordinal qn + 1)
                    tile_info<TR>(s_toff, s_seq, B, t, b, row0, row_end);
                    seq_end = s_toff[b + 1];
                    ++qn;
                    b_cur = b_desc0 + uint64_t(((qn & 1) * QIMG) >> 4);
                    if (!mbar_wait(&qfull[qn & 1], uint32_t((qn >> 1) & 1), abort_v, kWaitLimitNs)) break;
                }
                const int64_t gend = (seq_end < t1 ? seq_end : t1);
                const int gn = int(gend - t < G ? gend - t : G);
                uint64_t a_d[G];
                uint32_t d_t[G];
                int acc_of[G], st_of[G];   // accumulator and stage of each tile of the group
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    if (u >= gn) break;
                    if (!mbar_wait(&tempty[acc], aph ^ 1, abort_v, kWaitLimitNs)) { ok = false; break; }
                    if (!mbar_wait(&full[st], ph, abort_v, kWaitLimitNs)) { ok = false; break; }
                    a_d[u] = a_cur;
                    d_t[u] = tmem_base + uint32_t(acc * TILEC);
                    acc_of[u] = acc;
                    st_of[u] = st;
                    a_cur += kStageStep;
                    if (++st == S) { st = 0; ph ^= 1; a_cur = a_desc0; }
                    if (++acc == KACC) { acc = 0; aph ^= 1; }
                }
                if (!ok) break;
                t += gn;
                tc_fence_after();
                if (KIND == BF16_D128) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
#pragma unroll
                        for (int u = 0; u < G; ++u)
                            if (u < gn)
                                mma_f16(d_t[u], a_d[u] + uint64_t(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                                        b_cur + uint64_t(((kk >> 2) * (H * 128) + (kk & 3) * 32) >> 4), IDESC,
                                        kk > 0);
                } else if (KIND == BF16_D64) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                        for (int u = 0; u < G; ++u)
                            if (u < gn)
                                mma_f16(d_t[u], a_d[u] + uint64_t((kk * 32) >> 4), b_cur + uint64_t((kk * 32) >> 4),
                                        IDESC, kk > 0);
                } else if (KIND == E4M3_D64) {
                    // as below, with 64-byte rows: the halves are 8 KB apart, two K = 32 steps
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
#pragma unroll
                        for (int sub = 0; sub < 2; ++sub)
                            mma_f8(d_t[0] + uint32_t(sub * SUBC), a_d[0] + uint64_t((sub * 8192 + kk * 32) >> 4),
                                   b_cur + uint64_t((kk * 32) >> 4), IDESC, kk > 0);
                } else {
                    // the two 128-row halves of the tile (16 KB apart in the stage) into their own column
                    // blocks, chains interleaved; N = 2H covers both query pieces (piece 2's rows follow
                    // piece 1's in the operand)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                        for (int sub = 0; sub < 2; ++sub)
                            mma_f8(d_t[0] + uint32_t(sub * SUBC), a_d[0] + uint64_t((sub * 16384 + kk * 32) >> 4),
                                   b_cur + uint64_t((kk * 32) >> 4), IDESC, kk > 0);
                }
                issued = true;
#pragma unroll
                for (int u = 0; u < G; ++u)
                    if (u < gn) {
                        mma_commit(&tdone[acc_of[u]]);                  // accumulator ready
                        if (kStageDone) mma_commit(&tfree[st_of[u]]);   // stage free
                    }
                if (t == gend) mma_commit(&qrel[qn % kRel]);      // this sequence's operand is no longer read
            }
            if (issued) {
                // every issued MMA has finished before TMEM is released
                mma_commit(drain);
                volatile int no_abort = 0;
                if (!mbar_wait(drain, 0, &no_abort, kWaitLimitNs)) *abort_v = 1;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;              // 0..7
        const int grp = ew >> 2;              // warpgroup
        const int quarter = warp & 3;         // TMEM lanes 32*quarter .. +31
        // the warpgroups take alternate tiles, every sub-tile of a tile (one TMEM round trip)
        constexpr int kStep = kEpiGroups;
        const int64_t tfirst = t0 + grp;
        int b = 0, cur = -1, ord = -1, released = 0;
        int64_t row0, row_end;
        // a sequence ordinal this warp will not read again frees its slot (1 of the 8 epilogue arrivals)
        auto release_to = [&](int upto) {
            for (; released < upto; ++released)
                if (lane == 0) mbar_arrive(&qrel[released % kRel]);
        };
        if (nord > 0) {
            // the query operands of ordinals 0 and 1 (slots 0 and 1), built by all 8 epilogue warps
            // while the first keys load, so that no CTA's producer stalls at its first sequence change
            int bo = 0;
            int64_t r0, r1;
            tile_info<TR>(s_toff, s_seq, B, t0, bo, r0, r1);
            pdl_wait();   // the query and gate weights may come from the preceding kernel
            for (int o = 0; o < 2 && o < nord; ++o) {
                if (o == 1) {   // the next sequence that owns tiles
                    ++bo;
                    while (bo < B - 1 && s_toff[bo + 1] == s_toff[bo]) ++bo;
                }
                build_query<KIND, H>(q + size_t(bo) * H * d, w + size_t(bo) * H, d, qimg + o * QIMG, wsm + o * H,
                                     ew, kEpiWarps, lane);
                fence_proxy_async_smem();
                named_barrier(2, kEpiWarps * 32);
                if (ew == 0 && lane == 0) mbar_arrive(&qfull[o]);
            }
        }
        // ordinal of each tile: count the sequence changes over every tile of the range (both groups')
        int ob = 0, ocur = -1, onum = -1;
        int64_t orow0, orow1, u_next = t0;
        bool ok = true;
        for (int64_t t = tfirst; t < t1; t += kStep) {
            const int64_t i = t - t0;         // local tile index: accumulator i % KACC, its (i / KACC)-th use
            const int acc = int(i % KACC);
            const uint32_t aph = uint32_t((i / KACC) & 1);
            for (; u_next <= t; ++u_next) {
                tile_info<TR>(s_toff, s_seq, B, u_next, ob, orow0, orow1);
                if (ob != ocur) { ocur = ob; ++onum; }
            }
            tile_info<TR>(s_toff, s_seq, B, t, b, row0, row_end);
            if (b != cur) {
                cur = b;
                ord = onum;
                release_to(ord);   // earlier sequences: this warp is done with them
                // the gate weights of this sequence were written before the producer's arrival
                ok = mbar_wait(&qfull[ord & 1], uint32_t((ord >> 1) & 1), abort_v, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) break;
            }
            const float *wq = wsm + (ord & 1) * H;
            ok = mbar_wait(&tdone[acc], aph, abort_v, kWaitLimitNs);
            // the row scales landed long before (loaded with the keys); read before the release
            if (kScales) ok = ok && mbar_wait(&sfull[i % RS], uint32_t((i / RS) & 1), abort_v, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) break;   // keep the warp converged for tcgen05.ld
            tc_fence_after();
            // the tile's scales start at row0's offset from its aligned start when they came by bulk copy
            const int soff = (!LISTED && kScales && scales_bulk(row0, (row_end - row0) < TR ? (row_end - row0) : TR,
                                                                scale_len, k_scale))
                                 ? int(row0 & 3)
                                 : 0;
            const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(acc * TILEC);
            // the sub-tiles one after the other, each in chunks of up to 32 heads (both pieces' columns of a
            // chunk per TMEM round trip) through the same registers: a whole tile's row does not fit beside
            // the rest in the 168 registers of a 320-thread CTA; the accumulator is released once the last
            // chunk is in registers
            constexpr int HC = H < 32 ? H : 32;   // heads per chunk
            constexpr int NP = is_e4m3(KIND) ? 2 : 1;
            [[maybe_unused]] int kept = 0;   // fused selection: this warp's kept rows of the tile
#pragma unroll
            for (int sub = 0; sub < C::kSub; ++sub) {
                const float sc = kScales ? s_scale[int(i % RS) * SS + soff + sub * kRows + quarter * 32 + lane] : 1.f;
                float za = 0.f, zb = 0.f, zc = 0.f, zd = 0.f;   // four short dependency chains
#pragma unroll
                for (int h0 = 0; h0 < H; h0 += HC) {
                    uint32_t r[NP][HC];
#pragma unroll
                    for (int pc = 0; pc < NP; ++pc)
#pragma unroll
                        for (int c = 0; c < HC / 16; ++c)
                            tmem_ld_32x32b_x16(taddr + sub * SUBC + pc * H + h0 + c * 16,
                                               *reinterpret_cast<uint32_t(*)[16]>(&r[pc][c * 16]));
                    tmem_ld_wait();
                    if (sub == C::kSub - 1 && h0 + HC == H) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty[acc]);
                    }
#pragma unroll
                    for (int j = 0; j < HC; j += 4) {
                        const float4 wv = *reinterpret_cast<const float4 *>(wq + h0 + j);
                        float v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            v[e] = NP == 2 ? __uint_as_float(r[0][j + e]) + __uint_as_float(r[NP - 1][j + e])
                                           : __uint_as_float(r[0][j + e]);
                        za = fmaf(wv.x, fmaxf(v[0], 0.f), za);
                        zb = fmaf(wv.y, fmaxf(v[1], 0.f), zb);
                        zc = fmaf(wv.z, fmaxf(v[2], 0.f), zc);
                        zd = fmaf(wv.w, fmaxf(v[3], 0.f), zd);
                    }
                }
                float zs = (za + zb) + (zc + zd);
                if constexpr (SEL)
                    if (kScales) zs *= sc;
                const int64_t row = row0 + sub * kRows + quarter * 32 + lane;   // entry (full) or list position
                if (row < row_end) {
                    if constexpr (!SEL)
                        if (kScales) zs *= sc;
                    z[row] = zs;
                    if (I) I[row] = 1.f / (1.f + expf(-zs));
                }
                if constexpr (SEL) {
                    // fused selection (I >= 0.5 <=> z >= 0): bit `lane` of word 4 sub + quarter of tile t is
                    // row row0 + 128 sub + 32 quarter + lane
                    const uint32_t word = __ballot_sync(0xffffffffu, row < row_end && zs >= 0.f);
                    if (lane == 0) sel_bits[t * (4 * C::kSub) + 4 * sub + quarter] = word;
                    kept += __popc(word);
                }
            }
            if constexpr (SEL)
                if (lane == 0) sel_cnt[t * 4 + quarter] = kept;
        }
        release_to(nord);   // every sequence of the range
    }
    __syncwarp();   // lanes that skipped a role loop wait for their lane 0 here
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, NCOL);
    }
    if (threadIdx.x == 0 && *abort_v) raise_err(err, LSA_ERR_TIMEOUT);
}

// ------------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

template <int KIND, int H>
size_t smem_bytes(int B) {
    using C = Cfg<KIND>;
    return 1024 + size_t(C::kStages) * C::kStageBytes + 2 * qimg_bytes<KIND, H>() +
           (C::kStages + 2 + kRel + kDoneMax + kAccMax + 1 + kScaleSlotsMax) * 8 + 16 + 16 + 2 * H * 4 +
           size_t(B + 1) * 24 + 16 +
           (is_e4m3(KIND) ? size_t(C::kStages + acc_tiles<KIND, H>()) * (tile_rows<KIND>() + 8) * 4 : 0) +
           64;
}

struct ScanArgs {
    const void *q;
    const float *w;
    const void *k;
    const float *k_scale;
    const int64_t *seq_off;   // the tile axis of a full scan (sequence offsets, or a device-produced axis)
    int64_t n_total;          // rows of the key array
    const int32_t *idx;       // listed mode: entry lists (NULL: full mode)
    const int64_t *idx_off;
    int64_t list_cap;
    int B, d;
    float *z, *I;
    int32_t *err;
    int64_t axis_cap;         // full mode over a device-produced axis: its capacity (0: seq_off is constant)
    int64_t scale_len;        // entries of k_scale
    uint32_t *sel_bits = nullptr;   // fused selection (full mode): per tile, one ballot word per 32 rows
    int32_t *sel_cnt = nullptr;     // ... and the kept rows of each of its 4 row quarters
};

template <int KIND, int H>
lsa_status launch(const ScanArgs &a, cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) {
        set_error("lsa_index_score: cuTensorMapEncodeTiled is unavailable");
        return LSA_ERR_CUDA;
    }
    CUtensorMap map;
    const bool fp8 = is_e4m3(KIND);
    const cuuint64_t dims[2] = {cuuint64_t(a.d), cuuint64_t(a.n_total)};
    const cuuint64_t strides[1] = {cuuint64_t(a.d) * (fp8 ? 1 : 2)};
    // box: one 128-byte column block (64 bytes for e4m3 d = 64) x kBoxRows rows
    const cuuint32_t box[2] = {cuuint32_t(fp8 ? a.d : 64), cuuint32_t(Cfg<KIND>::kBoxRows)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void *>(a.k), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     KIND == E4M3_D64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("lsa_index_score: cuTensorMapEncodeTiled failed (%d)", int(r));
        return LSA_ERR_CUDA;
    }
    const size_t smem = smem_bytes<KIND, H>(a.B);
    auto kern = a.idx ? scan_tc<KIND, H, true> : (a.sel_bits ? scan_tc<KIND, H, false, true> : scan_tc<KIND, H, false>);
    LSA_CUDA(ensure_smem(kern, smem));
    const int64_t axis = a.idx ? a.list_cap : (a.axis_cap > 0 ? a.axis_cap : a.n_total);
    const int64_t max_tiles = (axis + tile_rows<KIND>() - 1) / tile_rows<KIND>() + a.B;
    const int grid = int(max_tiles < sm_count() ? max_tiles : sm_count());
    LSA_CUDA(launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, map, static_cast<const uint8_t *>(a.k),
                        static_cast<const uint16_t *>(a.q), a.w, a.d, a.seq_off, a.idx, a.idx_off, a.list_cap, a.B,
                        a.k_scale, a.scale_len, a.axis_cap, a.z, a.I, a.sel_bits, a.sel_cnt, a.err));
    static const char *kNames[2][4] = {
        {"scan_tc bf16 d128", "scan_tc bf16 d64", "scan_tc e4m3 d128", "scan_tc e4m3 d64"},
        {"scan_tc_listed bf16 d128", "scan_tc_listed bf16 d64", "scan_tc_listed e4m3 d128", "scan_tc_listed e4m3 d64"}};
    LSA_LAUNCHED(kNames[a.idx ? 1 : 0][KIND]);
    return LSA_OK;
}

template <int KIND>
lsa_status launch_h(int H, const ScanArgs &a, cudaStream_t st) {
    switch (H) {
    case 16: return launch<KIND, 16>(a, st);
    case 32: return launch<KIND, 32>(a, st);
    default: return launch<KIND, 64>(a, st);
    }
}

lsa_status launch_kind(lsa_dtype k_dtype, int H, const ScanArgs &a, cudaStream_t st) {
    if (k_dtype == LSA_E4M3 && a.d == 128) return launch_h<E4M3_D128>(H, a, st);
    if (k_dtype == LSA_E4M3) return launch_h<E4M3_D64>(H, a, st);
    if (a.d == 128) return launch_h<BF16_D128>(H, a, st);
    return launch_h<BF16_D64>(H, a, st);
}

}  // namespace

bool index_score_tc_supported(lsa_dtype q_dtype, lsa_dtype k_dtype, int64_t n_total, int32_t B, int32_t H,
                              int32_t d) {
    // (a TMA box never exceeds the key matrix: at least one tile of rows)
    if (q_dtype != LSA_BF16 || B > kMaxB) return false;
    if (n_total < (k_dtype == LSA_E4M3 ? tile_rows<E4M3_D128>() : kRows)) return false;
    if (!(H == 16 || H == 32 || H == 64)) return false;
    if (k_dtype == LSA_BF16 || k_dtype == LSA_E4M3) return d == 128 || d == 64;
    return false;
}

lsa_status launch_index_score_tc(const void *q, const float *w, const void *k, lsa_dtype k_dtype,
                                 const float *k_scale, const int64_t *seq_off, int64_t n_total,
                                 const int32_t *idx, const int64_t *idx_off, int64_t list_cap, int32_t B,
                                 int32_t H, int32_t d, float *z, float *I, int32_t *err, cudaStream_t st) {
    const ScanArgs a{q, w, k, k_scale, seq_off, n_total, idx, idx_off, list_cap, B, d, z, I, err, 0, n_total};
    return launch_kind(k_dtype, H, a, st);
}

int index_score_tc_tile_rows(lsa_dtype k_dtype) {
    return k_dtype == LSA_E4M3 ? tile_rows<E4M3_D128>() : tile_rows<BF16_D128>();
}

lsa_status launch_index_score_tc_select(const void *q, const float *w, const void *k, lsa_dtype k_dtype,
                                        const float *k_scale, const int64_t *seq_off, int64_t n_total, int32_t B,
                                        int32_t H, int32_t d, float *z, uint32_t *sel_bits, int32_t *sel_cnt,
                                        int32_t *err, cudaStream_t st) {
    ScanArgs a{q, w, k, k_scale, seq_off, n_total, nullptr, nullptr, 0, B, d, z, nullptr, err, 0, n_total};
    a.sel_bits = sel_bits;
    a.sel_cnt = sel_cnt;
    return launch_kind(k_dtype, H, a, st);
}

lsa_status launch_index_score_tc_axis(const void *q, const float *w, const void *k, lsa_dtype k_dtype,
                                      const float *k_scale, int64_t scale_len, const int64_t *axis_off,
                                      int64_t axis_cap, int64_t n_rows, int32_t B, int32_t H, int32_t d, float *z,
                                      int32_t *err, cudaStream_t st) {
    const ScanArgs a{q,  w,        k,    k_scale, axis_off, n_rows, nullptr, nullptr, 0, B, d, z, nullptr,
                     err, axis_cap, scale_len};
    return launch_kind(k_dtype, H, a, st);
}

}  // namespace lsa
