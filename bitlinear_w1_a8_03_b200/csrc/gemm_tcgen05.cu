// Ternary × int8 GEMM on the 5th-generation tensor cores (tcgen05), for the
// many-token (prefill) product.
//
// Computes the same acc[m][n] = Σ_k x̃[m][k]·Ŵ[n][k] as the GEMV (the pages'
// add / subtract / skip, "1.58 位大模型", nxmr.cn/news/148658 §3.3, carried out
// by the int8 tensor cores, which 2kiu.com/news/4928193 §3.3 names for the
// GEMM-shaped batched case) and the dequantisation y = fp32(acc)·α·β/127 +
// bias ("1.58-bit 大模型极限量化实战", chenxutan.com/d/5049.html §2.4–§2.5, §4.2).
//
// Persistent kernel, one CTA per SM.  A tile is 256 weight rows (two MMAs of
// M = 128 that share each x̃ tile, which halves the x̃ bytes per MAC) × NT
// tokens (the MMA's N side); K runs in blocks of 128.  Tiles are dealt
// round-robin to the CTAs.  Warp roles (15 warps):
//   warp 0      one thread loads x̃ tiles [NT tokens][128 B] by TMA (128-byte
//               swizzle) into ring B;
//   warp 10     one thread loads packed-code tiles [256 rows][32 B] by TMA
//               into ring W, running ahead of the tensor cores;
//   warps 2-5   expand the 2-bit codes of two rows each (rows t and 128 + t)
//               from ring W into signed bytes {-1, 0, +1} in ring A, laid out
//               K-major with the 128-byte swizzle the MMA descriptors expect;
//   warp 1      owns the tensor memory (the accumulators: two per tile, twice
//               over when they fit) and one thread issues
//               tcgen05.mma.kind::i8 (8 per K block) and the commits that free
//               ring slots / publish an accumulator;
//   warps 6-9,  epilogue: tcgen05.ld of a row's accumulators, scale by the
//   11-14       token's α·β/127, add bias, store (consecutive threads write
//               consecutive rows); the two groups take half of the token
//               columns each.
// For at most 64 tokens gemm_tm_kernel below is used instead.
// Every wait is bounded; on expiry the kernel records BL_ERR_TIMEOUT, the
// other roles stop at their next wait, copies and MMAs in flight drain
// (bounded) and the tensor memory is freed.
#include <cuda.h>

#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "bl_common.cuh"
#include "bl_launch.h"
#include "bl_ptx.cuh"

namespace bl {

static __device__ int g_gemm_error;

namespace {

constexpr int kKB = 128;          // K (bytes of x̃ = weights) per block
constexpr int kWB = kKB / 4;      // packed bytes of one row per K block
constexpr int kRowsTile = 128;    // weight rows per tile (MMA M)
constexpr int kWarps = 11;
constexpr int kThreads = kWarps * 32;
constexpr int kWarpTmaX = 0, kWarpMma = 1, kWarpExp0 = 2, kWarpEpi0 = 6, kWarpTmaW = 10;
constexpr int kExpWarps = 4, kEpiWarps = 4;
// the many-token kernel has a second group of four epilogue warps (11-14) that
// drains the other half of each accumulator's columns
constexpr int kWarpsTC = 15;
constexpr int kThreadsTC = kWarpsTC * 32;
constexpr int kEpiWarpsTC = 8;
constexpr size_t kSmemLimit = 232448;  // opt-in dynamic shared memory per block on sm_100

// Ring depths (expanded codes A, x̃ tiles B, packed codes W) for the two
// large tile widths; build-time knobs, the shared-memory budget is checked below.
#ifndef BL_GEMM_SA_256
#define BL_GEMM_SA_256 3
#endif
#ifndef BL_GEMM_SB_256
#define BL_GEMM_SB_256 3
#endif
#ifndef BL_GEMM_SW_256
#define BL_GEMM_SW_256 3
#endif
#ifndef BL_GEMM_SA_128
#define BL_GEMM_SA_128 4
#endif
#ifndef BL_GEMM_SB_128
#define BL_GEMM_SB_128 4
#endif
#ifndef BL_GEMM_SW_128
#define BL_GEMM_SW_128 4
#endif

// A tile is kHalves × 128 weight rows: two MMAs of M = 128 per K step share
// each x̃ (B) tile, which halves the x̃ bytes every MAC needs.
constexpr int kHalves = 2;
constexpr int kTileRows = kHalves * kRowsTile;

template <int NT>
struct Cfg {
    static constexpr int kAHalf = kRowsTile * kKB;     // 16 KiB of expanded codes per 128 rows
    static constexpr int kABytes = kHalves * kAHalf;    // the tile's rows
    static constexpr int kBBytes = NT * kKB;            // NT × 128 B of x̃
    static constexpr int kWBytes = kTileRows * kWB;     // packed codes of the tile's rows
    static constexpr int kSA = NT >= 256 ? BL_GEMM_SA_256 : BL_GEMM_SA_128;
    static constexpr int kSW = NT >= 256 ? BL_GEMM_SW_256 : BL_GEMM_SW_128;
    static constexpr int kSB = NT >= 256 ? BL_GEMM_SB_256 : BL_GEMM_SB_128;
    static constexpr int kBars = 2 * (kSA + kSB + kSW) + 5;
    // accumulators: kHalves × NT columns each; two of them when they fit
    static constexpr int kAccBufs = 2 * kHalves * NT <= 512 ? 2 : 1;
    static constexpr int kTmemCols = 512;
    static_assert(kAccBufs * kHalves * NT <= kTmemCols, "tensor memory budget");
    static constexpr size_t kRingBytes =
        (size_t)kSA * kABytes + (size_t)kSB * kBBytes + (size_t)kSW * kWBytes;
    static constexpr size_t kSmem = 1024 + kRingBytes + kBars * 8 + 16;
    static_assert(kSmem <= kSmemLimit, "shared memory budget");
    static_assert(kSmem > kSmemLimit / 2, "one CTA per SM (the tensor memory is sized for one)");
    static_assert(kSA >= 2 && kSB >= 2, "rings of at least two slots");
};

struct GemmProblem {
    const float* alpha;
    const float* beta;
    const float* bias;
    float* y;
    int32_t* acc_out;
    int M, N;
    int kblocks;
    int tiles_m;     // token tiles
    int tile_begin;  // first tile of this problem in the launch
};

// Several independent problems in one persistent launch: tiles are numbered
// problem after problem and dealt round-robin to the CTAs.
constexpr int kMaxListCtas = 256;
constexpr int kMaxListTiles = 2048;

struct GemmParams {
    CUtensorMap xmap[kMaxGroup];  // x̃ [M][K] of each problem
    CUtensorMap wmap[kMaxGroup];  // packed codes [N][row bytes] of each problem
    GemmProblem p[kMaxGroup];
    int count;
    int tiles;
    int cs;  // few-token kernel: CTAs per cluster, each taking 1/cs of every tile's K stages
    // many-token kernel: tiles of CTA c are tile_list[cta_start[c] .. cta_start[c+1])
    // (a longest-first greedy balance of K blocks), else round-robin
    int use_list;
    uint16_t cta_start[kMaxListCtas + 1];
    uint16_t tile_list[kMaxListTiles];
};

static_assert(sizeof(GemmParams) <= 32764, "kernel parameter block");

// The n-th tile of this CTA (or -1): from the host's list, else round-robin.
__device__ __forceinline__ int nth_tile(const GemmParams& P, int n) {
    if (P.use_list) {
        const int i = P.cta_start[blockIdx.x] + n;
        return i < P.cta_start[blockIdx.x + 1] ? P.tile_list[i] : -1;
    }
    const int64_t t = (int64_t)blockIdx.x + (int64_t)n * gridDim.x;
    return t < P.tiles ? (int)t : -1;
}

struct TileRef {
    int p, m0, n0, kblocks;
};

template <int NT, int ROWS = kRowsTile>
__device__ __forceinline__ TileRef locate(const GemmParams& P, int tile) {
    int p = 0;
    while (p + 1 < P.count && tile >= P.p[p + 1].tile_begin) ++p;
    const int local = tile - P.p[p].tile_begin;
    return TileRef{p, (local % P.p[p].tiles_m) * NT, (local / P.p[p].tiles_m) * ROWS, P.p[p].kblocks};
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart, tile base 1024-byte aligned.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);  // start address
    d |= (uint64_t)1 << 16;                 // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset
    d |= (uint64_t)1 << 46;                 // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                 // 128-byte swizzle
    return d;
}

// Instruction descriptor: s8 × s8 -> s32, A and B K-major, M = 128, N = NT.
template <int NT>
__host__ __device__ constexpr uint32_t instr_desc_i8() {
    return (2u << 4)            // D format s32
           | (1u << 7)          // A signed 8-bit
           | (1u << 10)         // B signed 8-bit
           | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(kRowsTile >> 4) << 24);
}

__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The mbarrier arrives once every tcgen05 operation this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive1(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Four signed bytes {-1, 0, +1} from the 2-bit codes of field s of a packed
// word: ((c | 0x80) - 1) ^ 0x80 per byte, with no borrow between bytes.
__device__ __forceinline__ uint32_t field_s8(uint32_t w, int s) {
    const uint32_t c = ((w >> (2 * s)) & 0x03030303u) | 0x80808080u;
    return (c - 0x01010101u) ^ 0x80808080u;
}

__device__ __forceinline__ void record_timeout(volatile int* abort_flag) {
    *abort_flag = 1;
    atomicCAS(&g_gemm_error, 0, (int)BL_ERR_TIMEOUT);
}

// Waits for phase `parity` of `bar` unless the CTA is aborting; false (and
// the abort recorded) if it did not complete.  A completed phase returns at
// once (one shared-memory access); the abort flag is read only when waiting.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_test_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (mbar_wait_bounded(bar, parity)) return true;
    record_timeout(abort_flag);
    return false;
}

// Both operands of one K block present: the two tests go out together.
__device__ __forceinline__ bool operands_ready(uint32_t bar_a, uint32_t par_a, uint32_t bar_b, uint32_t par_b,
                                               volatile int* abort_flag) {
    const bool a = mbar_test_wait(bar_a, par_a);
    const bool b = mbar_test_wait(bar_b, par_b);
    if (a & b) return true;
    return wait_or_abort(bar_a, par_a, abort_flag) && wait_or_abort(bar_b, par_b, abort_flag);
}

// A TMA producer's loop: one box per K block of every tile of this CTA into a
// ring of S slots, each reused once the consumer frees it.  On the way out it
// waits (bounded) for the copies it issued, so no copy lands after the CTA
// has exited.
template <int NT, int S, typename Coord>
__device__ void tma_producer(uint8_t* ring, uint32_t slot_bytes, uint64_t* full, uint64_t* empty,
                             const GemmParams& P, volatile int* abort_flag, Coord coord) {
    int it = 0;
    for (int n = 0, tile; (tile = nth_tile(P, n)) >= 0; ++n) {
        const TileRef tr = locate<NT, kTileRows>(P, tile);
        for (int kb = 0; kb < tr.kblocks; ++kb, ++it) {
            const int s = it % S;
            if (it >= S && !wait_or_abort(smem_addr(&empty[s]), ((it / S) - 1) & 1, abort_flag)) goto drain;
            int x, y;
            const CUtensorMap* map = coord(tr, kb, x, y);
            mbar_arrive_expect_tx(smem_addr(&full[s]), slot_bytes);
            tma_load_2d(smem_addr(ring + (size_t)s * slot_bytes), map, x, y, smem_addr(&full[s]));
        }
    }
drain:
    for (int j = it - 1; j >= 0 && j >= it - S; --j)
        if (!mbar_wait_bounded(smem_addr(&full[j % S]), (j / S) & 1)) record_timeout(abort_flag);
}

template <int NT>
__global__ void __launch_bounds__(kThreadsTC, 1) gemm_tc_kernel(const __grid_constant__ GemmParams P) {
    using C = Cfg<NT>;
    constexpr int SA = C::kSA, SB = C::kSB, SW = C::kSW;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* ringA = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ringB = ringA + (size_t)SA * C::kABytes;
    uint8_t* ringW = ringB + (size_t)SB * C::kBBytes;
    uint64_t* fullA = reinterpret_cast<uint64_t*>(ringW + (size_t)SW * C::kWBytes);
    uint64_t* emptyA = fullA + SA;
    uint64_t* fullB = emptyA + SA;
    // with equal ring depths one MMA commit releases A slot s and x̃ slot s
    // together (a commit costs the tensor pipe a few hundred cycles)
    constexpr bool kOneRelease = SA == SB;
    uint64_t* emptyB = kOneRelease ? emptyA : fullB + SB;
    uint64_t* fullW = fullB + 2 * SB;
    uint64_t* emptyW = fullW + SW;
    uint64_t* accFull = emptyW + SW;  // [2]
    uint64_t* accEmpty = accFull + 2;  // [2]
    uint64_t* drain = accEmpty + 2;    // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    constexpr int AB = C::kAccBufs;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    griddep_launch_dependents();  // a following PDL kernel may be scheduled; it waits for us

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(smem_addr(&fullA[s]), kExpWarps);
            mbar_init(smem_addr(&emptyA[s]), 1);
        }
        for (int s = 0; s < SB; ++s) {
            mbar_init(smem_addr(&fullB[s]), 1);
            if (!kOneRelease) mbar_init(smem_addr(&emptyB[s]), 1);
        }
        for (int s = 0; s < SW; ++s) {
            mbar_init(smem_addr(&fullW[s]), 1);
            mbar_init(smem_addr(&emptyW[s]), kExpWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_addr(&accFull[b]), 1);
            mbar_init(smem_addr(&accEmpty[b]), kEpiWarpsTC);
        }
        mbar_init(smem_addr(drain), 1);
        *abort_flag = 0;
    }
    fence_mbar_init();
    if (warp == kWarpMma) {  // tensor memory for the two accumulators
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(C::kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == kWarpTmaX) {
        // ---- x̃ tiles (written by the preceding kernel under PDL: wait for it first)
        if (lane == 0) {
            griddep_wait();
            tma_producer<NT, SB>(ringB, C::kBBytes, fullB, emptyB, P, abort_flag,
                                 [&](const TileRef& tr, int kb, int& x, int& y) {
                                     x = kb * kKB;
                                     y = tr.m0;
                                     return &P.xmap[tr.p];
                                 });
        }
    } else if (warp == kWarpTmaW) {
        // ---- packed codes (weights are not written by a kernel this launch may overlap)
        if (lane == 0)
            tma_producer<NT, SW>(ringW, C::kWBytes, fullW, emptyW, P, abort_flag,
                                 [&](const TileRef& tr, int kb, int& x, int& y) {
                                     x = kb * kWB;
                                     y = tr.n0;
                                     return &P.wmap[tr.p];
                                 });
    } else if (warp == kWarpMma) {
        // ---- MMA issue
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc_i8<NT>();
            int it = 0, j = 0;
            for (int tile; (tile = nth_tile(P, j)) >= 0; ++j) {
                const int kblocks = locate<NT, kTileRows>(P, tile).kblocks;
                const int b = j % AB;
                if (j >= AB && !wait_or_abort(smem_addr(&accEmpty[b]), ((j / AB) - 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_d + (uint32_t)(b * kHalves * NT);  // half h at + h·NT
                bool ok = true;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int sa = it % SA, sb = it % SB;
                    ok = operands_ready(smem_addr(&fullA[sa]), (it / SA) & 1, smem_addr(&fullB[sb]), (it / SB) & 1,
                                        abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t a_addr = smem_addr(ringA + (size_t)sa * C::kABytes);
                    const uint32_t b_addr = smem_addr(ringB + (size_t)sb * C::kBBytes);
#pragma unroll
                    for (int k = 0; k < kKB / 32; ++k)
#pragma unroll
                        for (int h = 0; h < kHalves; ++h)
                            mma_i8(d + (uint32_t)(h * NT), smem_desc_sw128(a_addr + h * C::kAHalf + 32 * k),
                                   smem_desc_sw128(b_addr + 32 * k), idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    mma_commit(smem_addr(&emptyA[sa]));
                    if constexpr (!kOneRelease) mma_commit(smem_addr(&emptyB[sb]));
                }
                if (!ok) break;
                mma_commit(smem_addr(&accFull[b]));
            }
            // every MMA issued above completes before the tensor memory is freed
            mma_commit(smem_addr(drain));
            if (!mbar_wait_bounded(smem_addr(drain), 0)) record_timeout(abort_flag);
        }
    } else if (warp < kWarpEpi0) {
        // ---- expand the codes of tile row t from ring W into ring A
        const int t = 32 * (warp & 3) + lane;
        const uint32_t a_row = (uint32_t)((t >> 3) * 1024 + (t & 7) * 128);
        int it = 0;
        for (int n = 0, tile; (tile = nth_tile(P, n)) >= 0; ++n) {
            const int kblocks = locate<NT, kTileRows>(P, tile).kblocks;
            bool ok = true;
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                const int sw = it % SW, sa = it % SA;
                if (!(ok = wait_or_abort(smem_addr(&fullW[sw]), (it / SW) & 1, abort_flag))) break;
                // rows t (first half) and 128 + t (second half) of the tile
                uint4 pk[kHalves][2];
#pragma unroll
                for (int h = 0; h < kHalves; ++h) {
                    const uint32_t wsrc =
                        smem_addr(ringW + (size_t)sw * C::kWBytes) + (uint32_t)(h * kRowsTile + t) * kWB;
                    pk[h][0] = lds128(wsrc);
                    pk[h][1] = lds128(wsrc + 16);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive1(smem_addr(&emptyW[sw]));  // codes are in registers
                if (it >= SA && !(ok = wait_or_abort(smem_addr(&emptyA[sa]), ((it / SA) - 1) & 1, abort_flag)))
                    break;
#pragma unroll
                for (int h = 0; h < kHalves; ++h) {
                    uint8_t* rowp = ringA + (size_t)sa * C::kABytes + h * C::kAHalf + a_row;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        // weights 16q .. 16q+15 of the block: fields 0..3 of packed word q
                        const uint32_t w = word_of(q < 4 ? pk[h][0] : pk[h][1], q & 3);
                        *reinterpret_cast<uint4*>(rowp + ((q ^ (t & 7)) << 4)) =
                            make_uint4(field_s8(w, 0), field_s8(w, 1), field_s8(w, 2), field_s8(w, 3));
                    }
                }
                fence_proxy_async_smem();  // generic writes -> tensor-core reads
                __syncwarp();
                if (lane == 0) mbar_arrive1(smem_addr(&fullA[sa]));
            }
            if (!ok) break;
        }
    } else {
        // ---- epilogue: tile row t (TMEM lane; a warp may only touch lanes 32·(warp % 4) .. +31)
        griddep_wait();  // β comes from, and y may be read by, the preceding kernel
        const int q = warp & 3;
        const int t = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int j = 0;
        for (int tile; (tile = nth_tile(P, j)) >= 0; ++j) {
            const TileRef tr = locate<NT, kTileRows>(P, tile);
            // this tile's problem, copied out of the parameter block once
            // (dynamically indexed parameter reads inside the store loop are slow)
            const int M = P.p[tr.p].M, N = P.p[tr.p].N;
            const float* beta_p = P.p[tr.p].beta;
            const float* bias_p = P.p[tr.p].bias;
            float* y = P.p[tr.p].y;
            int32_t* acc_out = P.p[tr.p].acc_out;
            const float alpha = *P.p[tr.p].alpha;
            const int b = j % AB;
            const int m0 = tr.m0;
            if (!wait_or_abort(smem_addr(&accFull[b]), (j / AB) & 1, abort_flag)) break;
            tc_fence_after();
            // warps 6-9 take the first half of the token columns, 11-14 the second
            const int cbeg = warp > kWarpTmaW ? NT / 2 : 0;
#pragma unroll 1
            for (int hh = 0; hh < kHalves; ++hh) {
                const int row = tr.n0 + hh * kRowsTile + t;
                const bool row_ok = row < N;
                const float bias = (row_ok && bias_p) ? bias_p[row] : 0.0f;
                const uint32_t col0 = (uint32_t)((b * kHalves + hh) * NT);
#pragma unroll 1
                for (int c0 = cbeg; c0 < cbeg + NT / 2; c0 += 32) {
                    // lane l holds the scale of token m0 + c0 + l; shuffled to the writers below
                    const int my_tok = m0 + c0 + lane;
                    const float my_scale = my_tok < M ? dequant_scale(alpha, beta_p[my_tok]) : 0.0f;
#pragma unroll
                    for (int h = 0; h < 2 && c0 + 16 * h < NT; ++h) {
                        uint32_t r[16];
                        tmem_ld16(tmem_d + lane_base + col0 + (uint32_t)(c0 + 16 * h), r);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float sc = __shfl_sync(0xffffffffu, my_scale, 16 * h + i);
                            const int tok = m0 + c0 + 16 * h + i;
                            if (row_ok && tok < M) {
                                const int acc = (int)r[i];
                                float out = __fmul_rn((float)acc, sc);
                                if (bias_p) out = __fadd_rn(out, bias);
                                y[(int64_t)tok * N + row] = out;
                                if (acc_out) acc_out[(int64_t)tok * N + row] = acc;
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive1(smem_addr(&accEmpty[b]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(C::kTmemCols));
    }
}

// ---------------------------------------------------------------- few tokens
// For at most 64 tokens the MMA is short (N = NT) and the shared-memory
// traffic of expanded code tiles, not the tensor pipe, sets the pace.  This
// variant expands the codes into TENSOR memory (tcgen05.st) and the MMA takes
// its A operand from there.  Codes stay unsigned, c = ŵ + 1 ∈ {0, 1, 2}
// (kind::i8 with A unsigned, B = x̃ signed), and TMEM lane 127 carries a row
// of ones, so D[t][m] = Σ_k c·x̃ and D[127][m] = Σ_k x̃: acc = D[t] - D[127],
// exact in int32.  A tile is 127 weight rows × NT tokens; K runs in stages of
// 512 (16 MMAs of 128×NT×32 per stage and barrier round trip).
namespace tm {
constexpr int kKS = 512;                // K per stage
constexpr int kWS = kKS / 4;            // packed bytes of one row per stage
constexpr int kRows = 127;              // weight rows per tile
constexpr int kOnes = 127;              // TMEM lane of the ones row
constexpr int kSA = 3;                  // A stages in tensor memory
constexpr uint32_t kACols = kKS / 4;    // 32-bit columns of one A stage
constexpr uint32_t kAccCols = 128;      // accumulators in columns [0, 2·NT)
constexpr uint32_t kTmemCols = 512;
static_assert(kAccCols + kSA * kACols <= kTmemCols, "tensor memory budget");
}  // namespace tm

template <int NT>
struct CfgTM {
    static constexpr int kWBytes = 128 * tm::kWS;  // a W slot: 127 rows × 128 B, 1024-aligned
    static constexpr int kWBox = tm::kRows * tm::kWS;
    static constexpr int kBBytes = NT * tm::kKS;   // four boxes of NT rows × 128 B
    static constexpr int kSW = NT >= 64 ? 5 : 6;
    static constexpr int kSB = tm::kSA;  // x̃ and A stages share one ring index and one release
    static constexpr int kBars = 2 * tm::kSA + 2 * kSW + 9;
    static constexpr int kRedStride = NT + 4;  // ints per row of the partial-sum buffer (conflict-free 16-byte access)
    static constexpr size_t kRedBytes = (size_t)128 * kRedStride * sizeof(int);
    static constexpr size_t kSmem = 1024 + (size_t)kSW * kWBytes + (size_t)kSB * kBBytes + kRedBytes + kBars * 8 + 16 +
                                    2 * NT * sizeof(int);
    static_assert(kSmem <= kSmemLimit, "shared memory budget");
    static_assert(kSmem > kSmemLimit / 2, "one CTA per SM (the tensor memory is sized for one)");
    static_assert(NT % 16 == 0 && 2 * NT <= (int)tm::kAccCols, "accumulator columns");
};

// Instruction descriptor: u8 (A, codes) × s8 (B, x̃) -> s32, both K-major, M = 128, N = NT.
template <int NT>
__host__ __device__ constexpr uint32_t instr_desc_u8s8() {
    return (2u << 4)  // D format s32
           | (0u << 7)  // A unsigned 8-bit
           | (1u << 10)  // B signed 8-bit
           | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(kRowsTile >> 4) << 24);
}

// MMA with A read from tensor memory (M rows in lanes 0..127, four 8-bit K
// elements per 32-bit column).
__device__ __forceinline__ void mma_i8_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// This thread's lane, 32 consecutive 32-bit columns from taddr.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---- thread-block clusters: split K between the CTAs of a cluster and sum
// the partial accumulators in the first CTA's shared memory
__device__ __forceinline__ bool mbar_test_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kPollSuspendNs)
        : "memory");
    return ok != 0;
}
// wait_or_abort for a barrier that threads of the other CTA of the cluster
// arrive on (their writes before the arrival are visible after it)
__device__ __forceinline__ bool wait_or_abort_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_test_wait_cluster(bar, parity)) return true;
    for (uint32_t i = 0; i < kPollLimit; ++i) {
        if (*abort_flag) return false;
        if (mbar_try_wait_cluster(bar, parity)) return true;
    }
    record_timeout(abort_flag);
    return false;
}
// The address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Every thread of every CTA of the cluster.  All paths through the kernel
// reach each call (every wait before it is bounded).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Stages [s0, s1) of a tile's S that CTA `rank` of a cs-CTA cluster takes.
__device__ __forceinline__ void stage_range(int S, int rank, int cs, int& s0, int& s1) {
    s0 = (rank * S) / cs;
    s1 = ((rank + 1) * S) / cs;
}

// A TMA producer that fills each ring slot with BOXES boxes (box b at
// slot + b·box_stride, all completing on the slot's barrier), over the tiles
// tile0, tile0 + tstep, … and stages [s0, s1) of each (this CTA's share).
template <int S, int BOXES, int ROWS, int NT, typename Coord>
__device__ void tma_producer_n(uint8_t* ring, uint32_t slot_bytes, uint32_t box_stride, uint32_t expect_bytes,
                               uint64_t* full, uint64_t* empty, const GemmParams& P, volatile int* abort_flag,
                               int tile0, int tstep, int rank, Coord coord) {
    int it = 0;
    for (int tile = tile0; tile < P.tiles; tile += tstep) {
        const TileRef tr = locate<NT, ROWS>(P, tile);
        int s0, s1;
        stage_range(tr.kblocks, rank, P.cs, s0, s1);
        for (int st = s0; st < s1; ++st, ++it) {
            const int s = it % S;
            if (it >= S && !wait_or_abort(smem_addr(&empty[s]), ((it / S) - 1) & 1, abort_flag)) goto drain;
            mbar_arrive_expect_tx(smem_addr(&full[s]), expect_bytes);
#pragma unroll
            for (int b = 0; b < BOXES; ++b) {
                int x, y;
                const CUtensorMap* map = coord(tr, st, b, x, y);
                tma_load_2d(smem_addr(ring + (size_t)s * slot_bytes + (size_t)b * box_stride), map, x, y,
                            smem_addr(&full[s]));
            }
        }
    }
drain:
    for (int j = it - 1; j >= 0 && j >= it - S; --j)
        if (!mbar_wait_bounded(smem_addr(&full[j % S]), (j / S) & 1)) record_timeout(abort_flag);
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) gemm_tm_kernel(const __grid_constant__ GemmParams P) {
    using C = CfgTM<NT>;
    constexpr int SA = tm::kSA, SB = C::kSB, SW = C::kSW;
    static_assert(SA == SB, "one ring index for the A and x̃ stages");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* ringW = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ringB = ringW + (size_t)SW * C::kWBytes;
    // A stage s (expander warps) and x̃ stage s (TMA) complete one barrier and
    // are released by one MMA commit (a commit costs the tensor pipe ~300 cycles)
    int* red_buf = reinterpret_cast<int*>(ringB + (size_t)SB * C::kBBytes);  // [128][kRedStride]: the partner's partial
    uint64_t* stageReady = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red_buf) + C::kRedBytes);
    uint64_t* stageFree = stageReady + SA;
    uint64_t* fullW = stageFree + SA;
    uint64_t* emptyW = fullW + SW;
    uint64_t* accFull = emptyW + SW;    // [2]
    uint64_t* accEmpty = accFull + 2;   // [2]
    uint64_t* onesReady = accEmpty + 2; // [2]
    uint64_t* partsIn = onesReady + 2;  // first CTA of a cluster: the second CTA's partial is in red_buf
    uint64_t* bufFree = partsIn + 1;    // second CTA: the first one has read red_buf
    uint64_t* drain = bufFree + 1;      // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* ones_sum = reinterpret_cast<int*>(tmem_slot + 4);  // [2][NT]: Σ x̃ of each token of the tile

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    griddep_launch_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(smem_addr(&stageReady[s]), kExpWarps + 1);
            mbar_init(smem_addr(&stageFree[s]), 1);
        }
        for (int s = 0; s < SW; ++s) {
            mbar_init(smem_addr(&fullW[s]), 1);
            mbar_init(smem_addr(&emptyW[s]), kExpWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_addr(&accFull[b]), 1);
            mbar_init(smem_addr(&accEmpty[b]), kEpiWarps);
            mbar_init(smem_addr(&onesReady[b]), 1);
        }
        mbar_init(smem_addr(partsIn), kEpiWarps * 32);
        mbar_init(smem_addr(bufFree), kEpiWarps * 32);
        mbar_init(smem_addr(drain), 1);
        *abort_flag = 0;
    }
    fence_mbar_init();
    if (warp == kWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(tm::kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;
    // cluster of cs CTAs (1 or 2): cluster cl takes tiles cl, cl + ncl, …; CTA
    // `rank` of it takes stages [rank·S/cs, (rank+1)·S/cs) of each
    const int cs = P.cs;
    const int rank = (int)(blockIdx.x % (unsigned)cs);
    const int cl = (int)(blockIdx.x / (unsigned)cs), ncl = (int)(gridDim.x / (unsigned)cs);
    if (cs > 1) cluster_sync_all();  // the partner's barriers are initialised before any remote arrive

    if (warp == kWarpTmaX) {
        // ---- x̃: four 128-byte boxes per stage (written by the preceding kernel under PDL)
        if (lane == 0) {
            griddep_wait();
            tma_producer_n<SB, 4, tm::kRows, NT>(ringB, C::kBBytes, NT * kKB, C::kBBytes, stageReady, stageFree, P, abort_flag,
                                                 cl, ncl, rank, [&](const TileRef& tr, int st, int b, int& x, int& y) {
                                                     x = st * tm::kKS + b * kKB;
                                                     y = tr.m0;
                                                     return &P.xmap[tr.p];
                                                 });
        }
    } else if (warp == kWarpTmaW) {
        // ---- packed codes: 127 rows × 128 B per stage (128-byte swizzle)
        if (lane == 0)
            tma_producer_n<SW, 1, tm::kRows, NT>(ringW, C::kWBytes, 0, C::kWBox, fullW, emptyW, P, abort_flag,
                                                 cl, ncl, rank, [&](const TileRef& tr, int st, int, int& x, int& y) {
                                                     x = st * tm::kWS;
                                                     y = tr.n0;
                                                     return &P.wmap[tr.p];
                                                 });
    } else if (warp == kWarpMma) {
        // ---- MMA issue: 16 per stage, A from tensor memory
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc_u8s8<NT>();
            int it = 0, j = 0;
            for (int tile = cl; tile < P.tiles; tile += ncl, ++j) {
                int s0, s1;
                stage_range(locate<NT, tm::kRows>(P, tile).kblocks, rank, cs, s0, s1);
                const int b = j & 1;
                if (j >= 2 && !wait_or_abort(smem_addr(&accEmpty[b]), ((j >> 1) - 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_d + (uint32_t)(b * NT);
                bool ok = true;
                for (int st = s0; st < s1; ++st, ++it) {
                    const int sa = it % SA;
                    if (!(ok = wait_or_abort(smem_addr(&stageReady[sa]), (it / SA) & 1, abort_flag))) break;
                    tc_fence_after();
                    const uint32_t a_col = tmem_d + tm::kAccCols + (uint32_t)sa * tm::kACols;
                    const uint32_t b_addr = smem_addr(ringB + (size_t)sa * C::kBBytes);
#pragma unroll
                    for (int k = 0; k < tm::kKS / 32; ++k)
                        mma_i8_ta(d, a_col + 8u * k, smem_desc_sw128(b_addr + (k >> 2) * (NT * kKB) + 32 * (k & 3)),
                                  idesc, (st > s0 || k > 0) ? 1u : 0u);
                    mma_commit(smem_addr(&stageFree[sa]));
                }
                if (!ok) break;
                mma_commit(smem_addr(&accFull[b]));
            }
            mma_commit(smem_addr(drain));
            if (!mbar_wait_bounded(smem_addr(drain), 0)) record_timeout(abort_flag);
        }
    } else if (warp < kWarpEpi0) {
        // ---- expand tile row t (= TMEM lane t) into the A stage; lane 127 is the ones row
        const int q = warp & 3;
        const int t = 32 * q + lane;
        const bool ones = t == tm::kOnes;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        // row t's 128 bytes, chunk j stored at chunk j ^ (t & 7) (128-byte swizzle)
        const uint32_t w_row = (uint32_t)t * tm::kWS;
        int it = 0;
        for (int tile = cl; tile < P.tiles; tile += ncl) {
            int s0, s1;
            stage_range(locate<NT, tm::kRows>(P, tile).kblocks, rank, cs, s0, s1);
            bool ok = true;
            for (int st = s0; st < s1; ++st, ++it) {
                const int sw = it % SW, sa = it % SA;
                if (!(ok = wait_or_abort(smem_addr(&fullW[sw]), (it / SW) & 1, abort_flag))) break;
                uint32_t wd[32];
                const uint32_t src = smem_addr(ringW + (size_t)sw * C::kWBytes) + w_row;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    // the ones row: 0x55 bytes hold code 1 in every field
                    const uint4 u = ones ? make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u)
                                         : lds128(src + 16u * (uint32_t)(c ^ (t & 7)));
                    wd[4 * c + 0] = u.x;
                    wd[4 * c + 1] = u.y;
                    wd[4 * c + 2] = u.z;
                    wd[4 * c + 3] = u.w;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive1(smem_addr(&emptyW[sw]));  // codes are in registers
                if (it >= SA && !(ok = wait_or_abort(smem_addr(&stageFree[sa]), ((it / SA) - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                const uint32_t a_col = tmem_d + lane_base + tm::kAccCols + (uint32_t)sa * tm::kACols;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    // word 8g + i holds weights 16(8g+i) .. +15; field f of it -> column 4(8g+i) + f
                    uint32_t r[32];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t w = wd[8 * g + i];
#pragma unroll
                        for (int f = 0; f < 4; ++f) r[4 * i + f] = (w >> (2 * f)) & 0x03030303u;
                    }
                    tmem_st32(a_col + 32u * g, r);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive1(smem_addr(&stageReady[sa]));
            }
            if (!ok) break;
        }
    } else {
        // ---- epilogue: tile row t; acc = D[t] - D[127] (with two CTAs per
        // cluster: the second sends its partial D to the first, which adds it)
        griddep_wait();
        const int q = warp & 3;
        const int t = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const uint32_t red_row = smem_addr(red_buf + t * C::kRedStride);
        int j = 0;
        for (int tile = cl; tile < P.tiles; tile += ncl, ++j) {
            const int b = j & 1;
            if (!wait_or_abort(smem_addr(&accFull[b]), (j >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            if (rank == 1) {
                // second CTA: once the first has read the previous partial, store
                // this row's partial into its buffer and tell it
                if (j > 0 && !wait_or_abort_cluster(smem_addr(bufFree), (j - 1) & 1, abort_flag)) break;
                const uint32_t dst = mapa_shared(red_row, 0);
#pragma unroll 1
                for (int c = 0; c < NT; c += 16) {
                    uint32_t r[16];
                    tmem_ld16(tmem_d + lane_base + (uint32_t)(b * NT + c), r);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        st_cluster_v4(dst + 4u * (uint32_t)(c + 4 * v), r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
                }
                mbar_arrive_remote(mapa_shared(smem_addr(partsIn), 0));
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive1(smem_addr(&accEmpty[b]));
                continue;
            }
            const bool add_part = cs > 1;
            if (add_part && !wait_or_abort_cluster(smem_addr(partsIn), j & 1, abort_flag)) break;
            const TileRef tr = locate<NT, tm::kRows>(P, tile);
            const int M = P.p[tr.p].M, N = P.p[tr.p].N;
            const float* beta_p = P.p[tr.p].beta;
            const float* bias_p = P.p[tr.p].bias;
            float* y = P.p[tr.p].y;
            int32_t* acc_out = P.p[tr.p].acc_out;
            const float alpha = *P.p[tr.p].alpha;
            const int m0 = tr.m0;
            const int row = tr.n0 + t;
            const bool row_ok = t < tm::kRows && row < N;
            const float bias = (row_ok && bias_p) ? bias_p[row] : 0.0f;
            int* ones_b = ones_sum + b * NT;
            if (q == 3) {
                // lane 31 of this warp reads TMEM lane 127: publish Σ x̃ of every token
#pragma unroll 1
                for (int c = 0; c < NT; c += 16) {
                    uint32_t r[16];
                    tmem_ld16(tmem_d + lane_base + (uint32_t)(b * NT + c), r);
                    if (lane == 31) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) ones_b[c + i] = (int)r[i] + (add_part ? red_buf[127 * C::kRedStride + c + i] : 0);
                    }
                }
                __syncwarp();
                if (lane == 31) mbar_arrive1(smem_addr(&onesReady[b]));
            }
            if (!wait_or_abort(smem_addr(&onesReady[b]), (j >> 1) & 1, abort_flag)) break;
#pragma unroll 1
            for (int c0 = 0; c0 < NT; c0 += 32) {
                const int my_tok = m0 + c0 + lane;
                const float my_scale = my_tok < M ? dequant_scale(alpha, beta_p[my_tok]) : 0.0f;
#pragma unroll
                for (int h = 0; h < 2 && c0 + 16 * h < NT; ++h) {
                    uint32_t r[16];
                    tmem_ld16(tmem_d + lane_base + (uint32_t)(b * NT + c0 + 16 * h), r);
                    if (add_part) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const uint4 u = lds128(red_row + 4u * (uint32_t)(c0 + 16 * h + 4 * v));
                            r[4 * v] += u.x;
                            r[4 * v + 1] += u.y;
                            r[4 * v + 2] += u.z;
                            r[4 * v + 3] += u.w;
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float sc = __shfl_sync(0xffffffffu, my_scale, 16 * h + i);
                        const int tok = m0 + c0 + 16 * h + i;
                        if (row_ok && tok < M) {
                            const int acc = (int)r[i] - ones_b[c0 + 16 * h + i];
                            float out = __fmul_rn((float)acc, sc);
                            if (bias_p) out = __fadd_rn(out, bias);
                            y[(int64_t)tok * N + row] = out;
                            if (acc_out) acc_out[(int64_t)tok * N + row] = acc;
                        }
                    }
                }
            }
            // red_buf row t has been read: the second CTA may overwrite it
            if (add_part) mbar_arrive_remote(mapa_shared(smem_addr(bufFree), 1));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive1(smem_addr(&accEmpty[b]));
        }
    }
    tc_fence_before();
    __syncthreads();
    // no CTA leaves while its partner may still write to or arrive in its shared memory
    if (cs > 1) cluster_sync_all();
    if (warp == kWarpMma) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(tm::kTmemCols));
    }
}


using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D uint8 tensor map over a row-major [rows][cols] array (row stride `cols`).
cudaError_t encode_u8(CUtensorMap* map, const void* base, int64_t cols, int64_t rows, uint32_t box_x, uint32_t box_y,
                      CUtensorMapSwizzle swizzle) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)cols};
    const cuuint32_t box[2] = {box_x, box_y};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The longest CTA's work, in stages (+1 per tile for the partial-sum exchange
// when cs = 2), with tiles dealt round-robin to `clusters` clusters of cs CTAs
// that split every tile's K stages.
int64_t split_makespan(const GemmParams& P, int clusters, int cs) {
    int64_t worst = 0;
    for (int c = 0; c < clusters; ++c) {
        int64_t sum = 0;
        int p = 0;
        for (int tile = c; tile < P.tiles; tile += clusters) {
            while (p + 1 < P.count && tile >= P.p[p + 1].tile_begin) ++p;
            sum += (P.p[p].kblocks + cs - 1) / cs + (cs > 1 ? 1 : 0);
        }
        worst = std::max(worst, sum);
    }
    return worst;
}

// Clusters of two CTAs of gemm_tm_kernel<NT> (one per SM) that the device
// can hold at once, cached per device.
template <int NT>
cudaError_t cluster_pairs(const void* kernel, int smem, int* out) {
    static std::mutex mu;
    static int cache[64] = {};  // per device: the count + 1 (0: not yet asked)
    int devi = 0;
    cudaError_t err = cudaGetDevice(&devi);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    if (devi < 64 && cache[devi] > 0) {
        *out = cache[devi] - 1;
        return cudaSuccess;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    err = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
    if (err != cudaSuccess) return err;
    if (devi < 64) cache[devi] = n + 1;
    *out = n;
    return cudaSuccess;
}

// Launches gemm_tc_kernel<NT> (TMEM_A = false: tiles of 128 rows, K blocks of
// 128, codes expanded in shared memory) or gemm_tm_kernel<NT> (TMEM_A = true:
// tiles of 127 rows, stages of 512, codes expanded in tensor memory).
template <int NT, bool TMEM_A>
cudaError_t launch_nt(const bitlinear_forward_problem* problems, int count, cudaStream_t stream, bool pdl) {
    constexpr int kRows = TMEM_A ? tm::kRows : kTileRows;
    constexpr int kStageK = TMEM_A ? tm::kKS : kKB;
    size_t kSmem;
    const void* kernel;
    if constexpr (TMEM_A) {
        kSmem = CfgTM<NT>::kSmem;
        kernel = reinterpret_cast<const void*>(gemm_tm_kernel<NT>);
    } else {
        kSmem = Cfg<NT>::kSmem;
        kernel = reinterpret_cast<const void*>(gemm_tc_kernel<NT>);
    }
    DeviceInfo dev;
    cudaError_t err = device_info(&dev);
    if (err != cudaSuccess) return err;
    // params are large (two tensor maps per problem): build them off the stack
    static thread_local GemmParams P;
    P = GemmParams{};
    P.count = count;
    // Tiles are numbered longest K first, so the round-robin deal hands out
    // the long tiles early and the short ones even out the end.
    int order[kMaxGroup];
    for (int i = 0; i < count; ++i) order[i] = i;
    std::stable_sort(order, order + count, [&](int a, int b) { return problems[a].K > problems[b].K; });
    int tiles = 0;
    for (int i = 0; i < count; ++i) {
        const bitlinear_forward_problem& pr = problems[order[i]];
        // Out-of-range boxes read zeros: a zero x̃ beyond K or beyond M, and
        // code 00 (-1) beyond a row's packed bytes or beyond N, which only
        // ever meets a zero x̃ or lands in a row that is not stored.
        err = encode_u8(&P.xmap[i], pr.x_q, pr.K, pr.M, kKB, NT, CU_TENSOR_MAP_SWIZZLE_128B);
        if (err != cudaSuccess) return err;
        const int64_t row_bytes = (int64_t)bitlinear_packed_row_bytes(pr.K);
        if (TMEM_A)
            err = encode_u8(&P.wmap[i], pr.W_packed, row_bytes, pr.N, tm::kWS, tm::kRows, CU_TENSOR_MAP_SWIZZLE_128B);
        else
            err = encode_u8(&P.wmap[i], pr.W_packed, row_bytes, pr.N, kWB, kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (err != cudaSuccess) return err;
        GemmProblem& q = P.p[i];
        q.alpha = pr.alpha;
        q.beta = pr.beta;
        q.bias = pr.bias;
        q.y = pr.y;
        q.acc_out = pr.acc_out;
        q.M = (int)pr.M;
        q.N = (int)pr.N;
        q.kblocks = (int)((pr.K + kStageK - 1) / kStageK);
        q.tiles_m = (int)((pr.M + NT - 1) / NT);
        q.tile_begin = tiles;
        tiles += q.tiles_m * (int)((pr.N + kRows - 1) / kRows);
    }
    P.tiles = tiles;
    P.cs = 1;
    P.use_list = 0;
    if constexpr (!TMEM_A) {
        // Longest-first greedy: each tile (numbered longest K first) goes to
        // the CTA with the fewest K blocks so far, so the CTAs end together
        // even when a few long tiles meet many short ones.
        const int G = tiles < dev.sm_count ? tiles : dev.sm_count;
        if (tiles <= kMaxListTiles && G <= kMaxListCtas) {
            static thread_local std::vector<std::pair<int64_t, int>> heap;
            static thread_local std::vector<int> owner;
            heap.clear();
            owner.assign((size_t)tiles, 0);
            for (int c = 0; c < G; ++c) heap.emplace_back(0, c);
            auto later = [](const std::pair<int64_t, int>& a, const std::pair<int64_t, int>& b) {
                return a.first != b.first ? a.first > b.first : a.second > b.second;
            };
            std::make_heap(heap.begin(), heap.end(), later);
            int p = 0;
            int count_per[kMaxListCtas] = {};
            for (int t = 0; t < tiles; ++t) {
                while (p + 1 < count && t >= P.p[p + 1].tile_begin) ++p;
                std::pop_heap(heap.begin(), heap.end(), later);
                auto& top = heap.back();
                owner[t] = top.second;
                ++count_per[top.second];
                top.first += P.p[p].kblocks;
                std::push_heap(heap.begin(), heap.end(), later);
            }
            P.cta_start[0] = 0;
            for (int c = 0; c < G; ++c) P.cta_start[c + 1] = (uint16_t)(P.cta_start[c] + count_per[c]);
            int fill[kMaxListCtas];
            for (int c = 0; c < G; ++c) fill[c] = P.cta_start[c];
            for (int t = 0; t < tiles; ++t) P.tile_list[fill[owner[t]]++] = (uint16_t)t;
            P.use_list = 1;
        }
    }

    // the opt-in is per device: set once on each device that launches the kernel
    err = set_max_dynamic_smem(kernel, (int)kSmem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(tiles < dev.sm_count ? tiles : dev.sm_count));
    cfg.blockDim = dim3(TMEM_A ? kThreads : kThreadsTC);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if constexpr (TMEM_A) {
        // Split every tile's K between the two CTAs of a cluster when that
        // shortens the longest CTA: few tiles for the SMs, long K.
        int ncl2 = 0;
        if (cluster_pairs<NT>(kernel, (int)kSmem, &ncl2) == cudaSuccess && ncl2 > 0) {
            int stages_min = INT32_MAX;
            for (int i = 0; i < count; ++i) stages_min = std::min(stages_min, P.p[i].kblocks);
            if (stages_min >= 2) {
                const int64_t one = split_makespan(P, std::min(tiles, dev.sm_count), 1);
                const int64_t two = split_makespan(P, std::min(tiles, ncl2), 2);
                if (two < one) {
                    P.cs = 2;
                    cfg.gridDim = dim3((unsigned)(2 * std::min(tiles, ncl2)));
                    attr[1].id = cudaLaunchAttributeClusterDimension;
                    attr[1].val.clusterDim.x = 2;
                    attr[1].val.clusterDim.y = 1;
                    attr[1].val.clusterDim.z = 1;
                    cfg.numAttrs = 2;
                }
            }
        }
    }
    void* args[] = {&P};
    return cudaLaunchKernelExC(&cfg, kernel, args);
}

}  // namespace

bool gemm_tc_supported(const bitlinear_forward_problem& p) {
    // TMA: x̃ rows (K bytes apart) and the x̃ base 16-byte aligned; tile counts in int
    return p.K % 16 == 0 && (reinterpret_cast<uintptr_t>(p.x_q) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(p.W_packed) & 15) == 0 && p.M <= ((int64_t)1 << 30) &&
           p.N <= ((int64_t)1 << 30) && ((p.M + 15) / 16) * ((p.N + kRowsTile - 1) / kRowsTile) < ((int64_t)1 << 26) &&
           encode_fn() != nullptr;
}

cudaError_t launch_gemm_tc(const bitlinear_forward_problem* problems, int count, cudaStream_t stream, bool pdl) {
    int64_t max_m = 0, tiles16 = 0;
    for (int i = 0; i < count; ++i) {
        max_m = problems[i].M > max_m ? problems[i].M : max_m;
        tiles16 += ((problems[i].M + 15) / 16) * ((problems[i].N + kRowsTile - 1) / kRowsTile);
    }
    if (tiles16 >= ((int64_t)1 << 30)) return cudaErrorInvalidValue;  // tile numbers are int
    if (max_m <= 16) return launch_nt<16, true>(problems, count, stream, pdl);
    if (max_m <= 32) return launch_nt<32, true>(problems, count, stream, pdl);
    if (max_m <= 64) return launch_nt<64, true>(problems, count, stream, pdl);
    if (max_m <= 128) return launch_nt<128, false>(problems, count, stream, pdl);
    return launch_nt<256, false>(problems, count, stream, pdl);
}

cudaError_t read_gemm_error(int* code) {
    int zero = 0;
    cudaError_t err = cudaMemcpyFromSymbol(code, g_gemm_error, sizeof(int));
    if (err != cudaSuccess) return err;
    return cudaMemcpyToSymbol(g_gemm_error, &zero, sizeof(int));
}

}  // namespace bl
