// Ternary × int8 GEMM on the 5th-generation tensor cores (tcgen05), for the
// many-token (prefill) product.
//
// Computes the same acc[m][n] = Σ_k x̃[m][k]·Ŵ[n][k] as the GEMV (the pages'
// add / subtract / skip, "1.58 位大模型", nxmr.cn/news/148658 §3.3, carried out
// by the int8 tensor cores, which 2kiu.com/news/4928193 §3.3 names for the
// GEMM-shaped batched case) and the dequantisation y = fp32(acc)·α·β/127 +
// bias ("1.58-bit 大模型极限量化实战", chenxutan.com/d/5049.html §2.4–§2.5, §4.2).
//
// Tile: 128 weight rows (the MMA's M side) × NT tokens (its N side) per CTA,
// K in blocks of 128.  Warp roles:
//   warp 0  one thread loads x̃ tiles [NT tokens][128 bytes] with TMA (128-byte
//           swizzle) into a ring of stages;
//   warp 1  owns the tensor memory (NT int32 columns) and one thread issues
//           tcgen05.mma.kind::i8 (4 per K block) and the commits that free a
//           stage / publish the accumulator;
//   warps 2-5 expand the 2-bit codes of their row (one row per thread) into
//           signed bytes {-1, 0, +1} in the UMMA K-major 128-byte-swizzled
//           layout, then run the epilogue: tcgen05.ld of the row's
//           accumulators, scale, store (consecutive threads = consecutive rows).
// Every wait is bounded; on expiry the kernel records BL_ERR_TIMEOUT, lets
// its copies and MMAs drain (bounded) and frees its tensor memory.
#include <cuda.h>

#include <mutex>

#include "bl_common.cuh"
#include "bl_launch.h"
#include "bl_ptx.cuh"

namespace bl {

static __device__ int g_gemm_error;

namespace {

constexpr int kKB = 128;          // K bytes (= weights) per block
constexpr int kRowsTile = 128;    // weight rows per tile (MMA M)
constexpr int kThreads = 6 * 32;  // producer, MMA, 4 expander/epilogue warps
constexpr int kExp = 128;         // expander threads

template <int NT>
struct Cfg {
    static constexpr int kStages = NT >= 256 ? 3 : 4;
    static constexpr int kABytes = kRowsTile * kKB;  // 16 KiB
    static constexpr int kBBytes = NT * kKB;         // NT × 128 B
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kTmemCols = NT < 32 ? 32 : NT;
};

struct GemmParams {
    const uint8_t* W;  // packed rows
    const float* alpha;
    const float* beta;
    const float* bias;
    float* y;
    int32_t* acc_out;
    int M, N, K;
    int row_bytes;
    int kblocks;
};

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

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                               const __grid_constant__ GemmParams P) {
    using C = Cfg<NT>;
    constexpr int S = C::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // stages first (each 1024-aligned), then barriers and small arrays
    uint8_t* stage_base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_b = reinterpret_cast<uint64_t*>(stage_base + S * C::kStageBytes);
    uint64_t* full_a = full_b + S;
    uint64_t* empty = full_a + S;
    uint64_t* acc_full = empty + S;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    float* scale_s = reinterpret_cast<float*>(tmem_slot + 4);  // [NT]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(scale_s + NT);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    griddep_launch_dependents();  // a following PDL kernel may be scheduled; it waits for us
    const int n0 = blockIdx.x * kRowsTile;
    const int m0 = blockIdx.y * NT;
    const int KB = P.kblocks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(&full_b[s]), 1);
            mbar_init(smem_addr(&full_a[s]), kExp / 32);
            mbar_init(smem_addr(&empty[s]), 1);
        }
        mbar_init(smem_addr(acc_full), 1);
        *abort_flag = 0;
    }
    fence_mbar_init();
    if (warp == 1) {  // tensor memory for the accumulator
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(C::kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    griddep_wait();  // x̃ and β may come from the preceding kernel
    if (threadIdx.x >= 64 && threadIdx.x < 64 + NT) {  // dequant scales of this tile's tokens
        const int t = threadIdx.x - 64;
        scale_s[t] = (m0 + t < P.M) ? dequant_scale(*P.alpha, P.beta[m0 + t]) : 0.0f;
    }
    if (NT > kExp && threadIdx.x >= 64) {
        for (int t = threadIdx.x - 64 + kExp; t < NT; t += kExp)
            scale_s[t] = (m0 + t < P.M) ? dequant_scale(*P.alpha, P.beta[m0 + t]) : 0.0f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        // ---- x̃ tiles by TMA
        if (lane == 0) {
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % S;
                if (kb >= S && !mbar_wait_bounded(smem_addr(&empty[s]), ((kb / S) - 1) & 1)) {
                    *abort_flag = 1;
                    atomicCAS(&g_gemm_error, 0, (int)BL_ERR_TIMEOUT);
                    break;
                }
                const uint32_t bar = smem_addr(&full_b[s]);
                mbar_arrive_expect_tx(bar, C::kBBytes);
                tma_load_2d(smem_addr(stage_base + s * C::kStageBytes + C::kABytes), &xmap, kb * kKB, m0, bar);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc_i8<NT>();
            bool ok = true;
            for (int kb = 0; kb < KB && ok; ++kb) {
                const int s = kb % S;
                ok = mbar_wait_bounded(smem_addr(&full_b[s]), (kb / S) & 1) &&
                     mbar_wait_bounded(smem_addr(&full_a[s]), (kb / S) & 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_addr = smem_addr(stage_base + s * C::kStageBytes);
                const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
                for (int k = 0; k < kKB / 32; ++k)
                    mma_i8(tmem_d, smem_desc_sw128(a_addr + 32 * k), smem_desc_sw128(b_addr + 32 * k), idesc,
                           (kb > 0 || k > 0) ? 1u : 0u);
                mma_commit(smem_addr(&empty[s]));
            }
            if (!ok) {
                *abort_flag = 1;
                atomicCAS(&g_gemm_error, 0, (int)BL_ERR_TIMEOUT);
            }
            mma_commit(smem_addr(acc_full));  // fires once every MMA issued above has completed
        }
    } else {
        // ---- expand the weight codes of row n0 + t, then the epilogue
        // tile row = TMEM lane; a warp may only touch lanes 32·(warp % 4) .. +31
        const int t = 32 * (warp & 3) + lane;
        const int row = n0 + t;
        const bool row_ok = row < P.N;
        const uint8_t* wrow = P.W + (int64_t)(row_ok ? row : 0) * P.row_bytes;
        const int chunks = P.row_bytes / 16;
        for (int kb = 0; kb < KB; ++kb) {
            const int s = kb % S;
            // packed codes of this K block: 2 chunks of 16 bytes (64 weights each)
            uint4 pk[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int ch = kb * 2 + h;
                pk[h] = (row_ok && ch < chunks) ? ld_stream16(wrow + 16 * ch)
                                                : make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
            }
            if (kb >= S && !mbar_wait_bounded(smem_addr(&empty[s]), ((kb / S) - 1) & 1)) {
                *abort_flag = 1;
                atomicCAS(&g_gemm_error, 0, (int)BL_ERR_TIMEOUT);
                break;
            }
            if (*abort_flag) break;
            uint8_t* a_tile = stage_base + s * C::kStageBytes;
            uint8_t* rowp = a_tile + (t >> 3) * 1024 + (t & 7) * 128;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t w = word_of(pk[h], q);  // weights 16·(4h+q) .. +15 of the block
                    const int j = 4 * h + q;               // 16-byte chunk of the 128-byte row
                    uint4 out;
                    out.x = field_s8(w, 0);
                    out.y = field_s8(w, 1);
                    out.z = field_s8(w, 2);
                    out.w = field_s8(w, 3);
                    *reinterpret_cast<uint4*>(rowp + ((j ^ (t & 7)) << 4)) = out;
                }
            }
            fence_proxy_async_smem();  // generic writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) mbar_arrive1(smem_addr(&full_a[s]));
        }
        // ---- epilogue: row n0 + t, tokens m0 .. m0+NT-1
        const bool done = mbar_wait_bounded(smem_addr(acc_full), 0);
        if (!done) atomicCAS(&g_gemm_error, 0, (int)BL_ERR_TIMEOUT);
        tc_fence_after();
        if (done && !*abort_flag) {
            const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
            const float b = (row_ok && P.bias) ? P.bias[row] : 0.0f;
#pragma unroll 1
            for (int c0 = 0; c0 < NT; c0 += 16) {
                uint32_t r[16];
                tmem_ld16(tmem_d + lane_base + c0, r);
                if (row_ok) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int tok = m0 + c0 + i;
                        if (tok < P.M) {
                            const int acc = (int)r[i];
                            float out = __fmul_rn((float)acc, scale_s[c0 + i]);
                            if (P.bias) out = __fadd_rn(out, b);
                            P.y[(int64_t)tok * P.N + row] = out;
                            if (P.acc_out) P.acc_out[(int64_t)tok * P.N + row] = acc;
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(C::kTmemCols));
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

template <int NT>
size_t smem_bytes() {
    using C = Cfg<NT>;
    return 1024 + (size_t)C::kStages * C::kStageBytes + (3 * C::kStages + 1) * 8 + 16 + NT * 4 + 16;
}

template <int NT>
cudaError_t launch_nt(const bitlinear_forward_problem& pr, cudaStream_t stream, bool pdl) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)pr.K, (cuuint64_t)pr.M};
    const cuuint64_t gstride[1] = {(cuuint64_t)pr.K};
    const cuuint32_t box[2] = {(cuuint32_t)kKB, (cuuint32_t)NT};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(pr.x_q), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    GemmParams P{};
    P.W = pr.W_packed;
    P.alpha = pr.alpha;
    P.beta = pr.beta;
    P.bias = pr.bias;
    P.y = pr.y;
    P.acc_out = pr.acc_out;
    P.M = (int)pr.M;
    P.N = (int)pr.N;
    P.K = (int)pr.K;
    P.row_bytes = (int)bitlinear_packed_row_bytes(pr.K);
    P.kblocks = (int)((pr.K + kKB - 1) / kKB);
    const size_t smem = smem_bytes<NT>();
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [smem] {
        attr_err = cudaFuncSetAttribute(gemm_tc_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (attr_err != cudaSuccess) return attr_err;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((pr.N + kRowsTile - 1) / kRowsTile), (unsigned)((pr.M + NT - 1) / NT));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<NT>, map, P);
}

}  // namespace

bool gemm_tc_supported(const bitlinear_forward_problem& p) {
    return p.K % 16 == 0 && (reinterpret_cast<uintptr_t>(p.x_q) & 15) == 0 && p.M <= ((int64_t)1 << 30) &&
           p.N <= ((int64_t)1 << 30) && encode_fn() != nullptr;
}

cudaError_t launch_gemm_tc(const bitlinear_forward_problem& p, cudaStream_t stream, bool pdl) {
    if (p.M <= 16) return launch_nt<16>(p, stream, pdl);
    if (p.M <= 32) return launch_nt<32>(p, stream, pdl);
    if (p.M <= 64) return launch_nt<64>(p, stream, pdl);
    if (p.M <= 128) return launch_nt<128>(p, stream, pdl);
    return launch_nt<256>(p, stream, pdl);
}

cudaError_t read_gemm_error(int* code) {
    int zero = 0;
    cudaError_t err = cudaMemcpyFromSymbol(code, g_gemm_error, sizeof(int));
    if (err != cudaSuccess) return err;
    return cudaMemcpyToSymbol(g_gemm_error, &zero, sizeof(int));
}

}  // namespace bl
