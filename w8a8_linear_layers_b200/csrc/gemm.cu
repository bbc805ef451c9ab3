// gemm.cu -- step 5: INT8 x INT8 -> INT32 GEMM with a fused per-token x
// per-output-channel dequantization epilogue, for sm_100a (B200).
//
// Source: CUDA INT8 quantization notes (aicoding.csdn.net), section 3.2
// ("低精度矩阵乘实现": an INT8 tensor-core matrix multiply, tiled, with
// double-buffered operand staging) and section 4.2 ("内核融合优化":
// quantize -> integer product -> dequantize fused in one kernel, persistent
// thread blocks).  The WMMA/Ampere kernel described there is prior art only;
// this kernel is built for the 5th-generation tensor cores:
//
//   * tcgen05.mma.cta_group::1.kind::i8, 128 x BN x 32 per instruction, int32
//     accumulators in tensor memory (TMEM), issued by one thread;
//   * operands staged by TMA (cp.async.bulk.tensor.2d, 128-byte swizzle,
//     zero fill past the matrix edges) into a STAGES-deep shared-memory ring
//     guarded by mbarriers (full: TMA bytes landed; empty: the MMAs that read
//     the stage completed, signalled by tcgen05.commit);
//   * persistent CTAs (one per SM) walking the output tiles; two TMEM
//     accumulator buffers so the epilogue of one tile overlaps the main loop
//     of the next;
//   * warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer,
//     then epilogue warps (TMEM lanes 32*(warp%4) .. +31 each).
//
// Four kernels share these pieces: w8a8_gemm_kernel (one CTA per 128 x 256
// tile, 64 < M <= 128), w8a8_gemm_pair_kernel (CTA pairs, cta_group::2,
// 256 x 256 tiles, 8 epilogue warps, M > 128), w4a8_gemm_kernel (packed int4
// weights unpacked on chip by converter warps, M > 64) and, for M <= 64,
// w8a8_gemm_decode_kernel (gemm_decode.cuh: weights as the 128-row operand,
// K split over a cluster where the weight tiles are few).
//
// Epilogue: tcgen05.ld of 32 accumulator columns per thread (thread = output
// row), y = ((float)acc * sx[row]) * sw[col] (two fp32 multiplies, int->fp32
// round-to-nearest-even), or with asymmetric weights
// sx * (sw * (float)(acc + 128 R) + ow * (float)R), converted to bf16 (RNE) or
// kept fp32, and stored: by the pair kernel through a 128B-swizzled
// shared-memory buffer and TMA stores (32 rows x 128 bytes a warp), by the
// others with 16-byte stores.  Optionally the raw int32
// accumulators are stored too.
//
// No TMA multicast is used anywhere (each CTA loads its own tiles).
//
// Every mbarrier wait is bounded: after kWaitNs without progress the waiting
// thread records a fault code in a device word (read by sq_device_fault),
// raises a CTA-wide abort flag, and every role leaves its loop; in-flight TMA
// copies and MMAs are drained (again with a bound) before TMEM is freed and
// the kernel returns.  Nothing traps.
#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace w8a8 {

__device__ unsigned int g_gemm_fault;

namespace gemm {

constexpr int BM = 128;          // rows of X per tile (= MMA M, = TMEM lanes)
constexpr int BK = 128;          // K bytes per stage (one 128-byte swizzle row)
constexpr int UMMA_K = 32;       // K per tcgen05.mma of kind::i8
constexpr int kThreads = 192;    // 6 warps
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s

enum : unsigned {
    kFaultProducer = 1,
    kFaultMmaFull = 2,
    kFaultMmaTmemEmpty = 3,
    kFaultEpilogue = 4,
    kFaultDrain = 5,
    kFaultSelftest = 6,
    kFaultConvert = 7,
};

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the phase of `bar` with the given parity.  Returns false
// if the CTA aborted (this thread timed out, or another role did).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             unsigned code, unsigned long long limit_ns = kWaitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            atomicCAS(&g_gemm_fault, 0u, code);
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy accesses (TMA stores, tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same MMA with the A operand (M = 128 rows, K-major, four int8 per
// 32-bit column) read from tensor memory at column a_tmem.
__device__ __forceinline__ void mma_i8_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05 op this thread issued so far completes.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane from registers
// (warp-collective), then wait until the stores are done.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzle: rows of 128 bytes, 8-row core groups 1024 bytes
// apart (stride byte offset), leading byte offset unused for swizzled
// K-major (encoded 1), descriptor version 1 (sm_100), layout 2 = 128B swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3fffu);        // start address
    d |= (uint64_t)1u << 16;                       // leading byte offset (16 B units)
    d |= (uint64_t)(1024u >> 4) << 32;             // stride byte offset (16 B units)
    d |= (uint64_t)1u << 46;                       // version
    d |= (uint64_t)2u << 61;                       // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::i8: D int32, A and B signed int8, both
// K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_i8(int m, int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

template <int BN>
struct Cfg {
    static constexpr int STAGES = 4;
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = 2 * BN;  // two accumulator buffers
    static constexpr int SMEM = STAGES * STAGE_BYTES + 1024;  // + alignment slack
    static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
};

// Dequant of one accumulator.  Symmetric weights: ((float)acc * sx) * sw.
// Asymmetric weights (w ~ sw (q + 128) + ow): with R the row sum of the
// activation codes and A = acc + 128 R (exact int32),
// sx * (sw * (float)A + ow * (float)R).
template <bool ASYM>
__device__ __forceinline__ float dequant1(uint32_t acc, float sxr, int Rr, float swv, float owv) {
    if (ASYM) {
        const float p = swv * __int2float_rn((int)acc + 128 * Rr);
        const float o = owv * __int2float_rn(Rr);
        return sxr * (p + o);
    }
    return (__int2float_rn((int)acc) * sxr) * swv;
}

template <typename OutT, bool ASYM>
__device__ __forceinline__ void store_row_chunk(OutT *yrow, const uint32_t (&acc)[32], float sxr, int Rr,
                                                const float *__restrict__ swc, const float *__restrict__ owc,
                                                int valid, bool vec_ok) {
    if (vec_ok && valid >= 32) {
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(swc + j));
            const float4 o = ASYM ? __ldg(reinterpret_cast<const float4 *>(owc + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
            y[j] = dequant1<ASYM>(acc[j], sxr, Rr, f.x, o.x);
            y[j + 1] = dequant1<ASYM>(acc[j + 1], sxr, Rr, f.y, o.y);
            y[j + 2] = dequant1<ASYM>(acc[j + 2], sxr, Rr, f.z, o.z);
            y[j + 3] = dequant1<ASYM>(acc[j + 3], sxr, Rr, f.w, o.w);
        }
        if (sizeof(OutT) == 2) {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                __nv_bfloat162 h = __floats2bfloat162_rn(y[j], y[j + 1]);
                packed[j / 2] = *reinterpret_cast<uint32_t *>(&h);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(yrow);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        } else {
            float4 *dst = reinterpret_cast<float4 *>(yrow);
#pragma unroll
            for (int j = 0; j < 32; j += 4) dst[j / 4] = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < valid) {
                const float v = dequant1<ASYM>(acc[j], sxr, Rr, swc[j], ASYM ? owc[j] : 0.0f);
                if (sizeof(OutT) == 2)
                    reinterpret_cast<__nv_bfloat16 *>(yrow)[j] = __float2bfloat16_rn(v);
                else
                    reinterpret_cast<float *>(yrow)[j] = v;
            }
    }
}

template <int BN, typename OutT, bool ASYM>
__global__ void __launch_bounds__(kThreads, 1)
w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const float *__restrict__ sx, const float *__restrict__ sw, const int32_t *__restrict__ rs,
                 const float *__restrict__ ow, OutT *__restrict__ y, int32_t *__restrict__ acc_out, int M, int N,
                 int K) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[C::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // 1024-aligned for 128B swizzle

    const int tiles_m = (M + BM - 1) / BM;
    const int tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int num_kb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tfull_bar[b]), 1);
            mbar_init(smem_u32(&tempty_bar[b]), 4 * 32);
        }
        mbar_init(smem_u32(&drain_bar), 1);
        abort_flag = 0;
        fence_barrier_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_a) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_b) : "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    pdl_wait();     // the codes and scales come from the previous kernel (prologue above overlapped it)
    pdl_trigger();  // the next kernel may launch; it waits for this grid before touching memory

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;  // stages whose loads were issued (for the abort drain)
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m0 = (tile % tiles_m) * BM, n0 = (tile / tiles_m) * BN;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, &abort_flag, kFaultProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_base + stage * C::STAGE_BYTES;
                    const uint32_t b_dst = a_dst + C::A_BYTES;
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
                    tma_load_2d(a_dst, &tmap_a, fb, kb * BK, m0);
                    tma_load_2d(b_dst, &tmap_b, fb, kb * BK, n0);
                    ++issued;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // drain: wait (bounded) for the copies of the last issued stages
                int outstanding = issued < C::STAGES ? issued : C::STAGES;
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < outstanding; ++i) {
                    if (--s < 0) {
                        s = C::STAGES - 1;
                        ph ^= 1u;
                    }
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try_wait(smem_u32(&full_bar[s]), ph) && globaltimer() - t0 < kWaitNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t buf_phase = 0;
            bool ok = true;
            bool issued_any = false;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!wait_bounded(smem_u32(&tempty_bar[buf]), buf_phase ^ 1u, &abort_flag, kFaultMmaTmemEmpty)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!wait_bounded(smem_u32(&full_bar[stage]), phase, &abort_flag, kFaultMmaFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_base + stage * C::STAGE_BYTES;
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        mma_i8(d_tmem, smem_desc_sw128(a_addr + k * UMMA_K), smem_desc_sw128(b_addr + k * UMMA_K),
                               idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    issued_any = true;
                    mma_commit(smem_u32(&empty_bar[stage]));
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(smem_u32(&tfull_bar[buf]));
                buf ^= 1;
                if (buf == 0) buf_phase ^= 1u;
            }
            if (!ok && issued_any) {
                // drain: every MMA issued so far completes before TMEM is freed
                mma_commit(smem_u32(&drain_bar));
                const unsigned long long t0 = globaltimer();
                while (!mbar_try_wait(smem_u32(&drain_bar), 0) && globaltimer() - t0 < kWaitNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int row_in_tile = quarter * 32 + lane;
        const bool vec_ok = (N % (16 / (int)sizeof(OutT))) == 0;
        const bool acc_vec_ok = (N % 4) == 0;
        int buf = 0;
        uint32_t buf_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int m0 = (tile % tiles_m) * BM, n0 = (tile / tiles_m) * BN;
            const int row = m0 + row_in_tile;
            const float sxr = row < M ? sx[row] : 0.0f;
            const int Rr = (ASYM && row < M) ? rs[row] : 0;
            // the TMEM loads below are warp-collective: leave together or not at all
            const bool ok = wait_bounded(smem_u32(&tfull_bar[buf]), buf_phase, &abort_flag, kFaultEpilogue);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t acc[32];
                tmem_ld32(tbase + (uint32_t)c0, acc);  // warp-collective: every lane takes part
                const int col = n0 + c0;
                if (row < M && col < N) {
                    const int valid = N - col;
                    OutT *yrow = y + (int64_t)row * N + col;
                    store_row_chunk<OutT, ASYM>(yrow, acc, sxr, Rr, sw + col, ASYM ? ow + col : nullptr, valid,
                                                vec_ok);
                    if (acc_out) {
                        int32_t *arow = acc_out + (int64_t)row * N + col;
                        if (acc_vec_ok && valid >= 32) {
#pragma unroll
                            for (int j = 0; j < 32; j += 4)
                                *reinterpret_cast<int4 *>(arow + j) =
                                    make_int4((int)acc[j], (int)acc[j + 1], (int)acc[j + 2], (int)acc[j + 3]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (j < valid) arow[j] = (int)acc[j];
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty_bar[buf]));
            buf ^= 1;
            if (buf == 0) buf_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ============================================================ 2-CTA pair kernel
// A cluster of two CTAs (a "pair") computes a 256 x 256 output tile with
// tcgen05.mma.cta_group::2: each CTA stages 128 rows of A (its half of the
// tile's M) and 128 rows of B (its half of N) per stage, and the pair's
// tensor cores compute 128 x 256 each into their own TMEM, reading both B
// halves.  Per SM this halves the B operand traffic of a 1-CTA 128 x 256 tile
// (64 instead of 96 shared-memory bytes per MMA cycle) and doubles the work
// each staged byte feeds.
//
// Synchronisation (leader = CTA rank 0 of the pair):
//   full[s]   (leader) : leader's producer posts arrive.expect_tx for both
//                        CTAs' bytes; both CTAs' TMA loads complete_tx on it;
//   empty[s]  (each)   : the leader's MMA commit multicasts to both CTAs;
//   tfull[b]  (each)   : the leader's commit after a tile's last k-block,
//                        multicast to both CTAs;
//   tempty[b] (leader) : all 2 x 128 epilogue threads of the pair arrive.
// TMEM (512 columns) is allocated and freed by warp 1 of both CTAs
// (cta_group::2); cluster barriers order barrier init before any remote
// arrival and keep both CTAs alive until the pair is done.

constexpr uint32_t kPeerMask = 0xFEFFFFFFu;  // shared::cluster address -> same offset in rank 0

// Tile t -> (m tile, n tile).  Consecutive pairs walk down M within a band of
// N tiles, so concurrently running pairs share B tiles in L2.
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int &tm, int &tn) {
#ifdef W8A8_TILE_N_FASTEST
    tm = tile / tiles_n;
    tn = tile % tiles_n;
#else
    tm = tile % tiles_m;
    tn = tile / tiles_m;
    (void)tiles_n;
#endif
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, uint32_t leader_bar, int x,
                                                 int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(dst),
        "l"((uint64_t)map), "r"(leader_bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` (same offset) in both CTAs of the pair once this thread's
// issued tcgen05 ops complete.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}"
        ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_leader(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar & kPeerMask) : "memory");
}

// SHIFT: the accumulator holds 2^SHIFT times the product (int4 operands, see
// unpack_int4x8) and is shifted back first.
template <typename OutT, bool ASYM, int SHIFT = 0>
__device__ __forceinline__ void epilogue_tile(uint32_t tbase, int row, int M, int n0, int N, const float sxr,
                                              int Rr, const float *__restrict__ sw, const float *__restrict__ ow,
                                              OutT *__restrict__ y, int32_t *__restrict__ acc_out, int BNc) {
    const bool vec_ok = (N % (16 / (int)sizeof(OutT))) == 0;
    const bool acc_vec_ok = (N % 4) == 0;
#pragma unroll 1
    for (int c0 = 0; c0 < BNc; c0 += 32) {
        uint32_t acc[32];
        tmem_ld32(tbase + (uint32_t)c0, acc);  // warp-collective
        if (SHIFT) {
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = (uint32_t)((int32_t)acc[j] >> SHIFT);  // exact: a multiple of 2^SHIFT
        }
        const int col = n0 + c0;
        if (row < M && col < N) {
            const int valid = N - col;
            store_row_chunk<OutT, ASYM>(y + (int64_t)row * N + col, acc, sxr, Rr, sw + col,
                                        ASYM ? ow + col : nullptr, valid, vec_ok);
            if (acc_out) {
                int32_t *arow = acc_out + (int64_t)row * N + col;
                if (acc_vec_ok && valid >= 32) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<int4 *>(arow + j) =
                            make_int4((int)acc[j], (int)acc[j + 1], (int)acc[j + 2], (int)acc[j + 3]);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < valid) arow[j] = (int)acc[j];
                }
            }
        }
    }
}

#ifndef W8A8_PAIR_STAGES
#define W8A8_PAIR_STAGES 6
#endif

#ifndef W8A8_PAIR_EPI_WARPS
#define W8A8_PAIR_EPI_WARPS 8
#endif
// Epilogue warps of the pair kernel: 4 cover the 128 TMEM lanes once; 8 split
// each tile's 256 columns between two warps per lane quarter, so that a short
// main loop (small K) does not wait on the epilogue.
constexpr int kPairEpiWarps = W8A8_PAIR_EPI_WARPS;
constexpr int kThreadsPair = 64 + 32 * kPairEpiWarps;

struct Cfg2 {
    static constexpr int BN = 256;              // pair tile N (each CTA stages BN/2 rows of B)
    static constexpr int PM = 2 * BM;           // pair tile M
    static constexpr int STAGES = W8A8_PAIR_STAGES;
    static constexpr int A_BYTES = BM * BK;     // 16 KB: this CTA's 128 rows of A
    static constexpr int B_BYTES = (BN / 2) * BK;  // 16 KB: this CTA's half of B
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = 2 * BN;    // two 128 x 256 accumulator buffers
    static constexpr int OUT_BYTES = 32 * 128;  // per epilogue warp: 32 rows x 128 bytes of output
    static constexpr int OUT_OFFSET = STAGES * STAGE_BYTES;
    static constexpr int SMEM = OUT_OFFSET + kPairEpiWarps * OUT_BYTES + 1024;
};

// TMA store of a 2-D box from shared memory, tracked by this thread's bulk
// groups; waits on the groups this thread committed.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"((uint64_t)map),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One 32-row chunk of a warp's output, staged and stored by TMA: the 32
// lanes' rows (lane = TMEM lane = output row) of CW = 128 / sizeof(OutT)
// columns from TMEM at taddr, dequantized, packed into the 128B-swizzled
// layout of the output tensor map's box (16-byte piece c of row r at piece
// c ^ (r & 7)), fenced to the async proxy and stored at (col, row0) by
// lane 0.  Columns past N read no scale and are clipped by the store, as are
// rows past M; a box wholly past either edge is skipped.  `pending`: lane 0
// has a store that may still read the buffer.
template <typename OutT, bool ASYM>
__device__ __forceinline__ void store_chunk_tma(const CUtensorMap *tmap_y, uint32_t taddr, uint32_t buf,
                                                int lane, int col, int row0, int M, int N, float sxr, int Rr,
                                                const float *__restrict__ sw, const float *__restrict__ ow,
                                                bool &pending) {
    constexpr int CW = 128 / (int)sizeof(OutT);
    if (col >= N || row0 >= M) return;  // warp-uniform: the whole box lies past the output
    uint32_t acc[CW];
    tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&acc[0]));
    if (CW == 64) tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&acc[CW == 64 ? 32 : 0]));
    uint32_t packed[32];
    const bool full = col + CW <= N;
#pragma unroll
    for (int j = 0; j < CW; j += 4) {
        float4 f, o = make_float4(0.f, 0.f, 0.f, 0.f);
        if (full) {
            f = __ldg(reinterpret_cast<const float4 *>(sw + col + j));
            if (ASYM) o = __ldg(reinterpret_cast<const float4 *>(ow + col + j));
        } else {
            f.x = col + j < N ? sw[col + j] : 0.f;
            f.y = col + j + 1 < N ? sw[col + j + 1] : 0.f;
            f.z = col + j + 2 < N ? sw[col + j + 2] : 0.f;
            f.w = col + j + 3 < N ? sw[col + j + 3] : 0.f;
            if (ASYM) {
                o.x = col + j < N ? ow[col + j] : 0.f;
                o.y = col + j + 1 < N ? ow[col + j + 1] : 0.f;
                o.z = col + j + 2 < N ? ow[col + j + 2] : 0.f;
                o.w = col + j + 3 < N ? ow[col + j + 3] : 0.f;
            }
        }
        const float v0 = dequant1<ASYM>(acc[j], sxr, Rr, f.x, o.x), v1 = dequant1<ASYM>(acc[j + 1], sxr, Rr, f.y, o.y);
        const float v2 = dequant1<ASYM>(acc[j + 2], sxr, Rr, f.z, o.z), v3 = dequant1<ASYM>(acc[j + 3], sxr, Rr, f.w, o.w);
        if (sizeof(OutT) == 2) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(v0, v1), hi = __floats2bfloat162_rn(v2, v3);
            packed[j / 2] = *reinterpret_cast<uint32_t *>(&lo);
            packed[j / 2 + 1] = *reinterpret_cast<uint32_t *>(&hi);
        } else {
            packed[j] = __float_as_uint(v0);
            packed[j + 1] = __float_as_uint(v1);
            packed[j + 2] = __float_as_uint(v2);
            packed[j + 3] = __float_as_uint(v3);
        }
    }
    if (lane == 0 && pending) bulk_wait_read_all();  // the previous store has read the buffer
    __syncwarp();
    const uint32_t rowp = buf + (uint32_t)lane * 128u;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowp + (uint32_t)(((c ^ (lane & 7)) << 4))),
                     "r"(packed[4 * c]), "r"(packed[4 * c + 1]), "r"(packed[4 * c + 2]), "r"(packed[4 * c + 3])
                     : "memory");
    fence_proxy_async_smem();  // the TMA store reads these bytes through the async proxy
    __syncwarp();
    if (lane == 0) tma_store_2d(tmap_y, buf, col, row0);
    pending = true;
}

template <typename OutT, bool ASYM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsPair, 1)
w8a8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_y, const float *__restrict__ sx, const float *__restrict__ sw, const int32_t *__restrict__ rs,
                      const float *__restrict__ ow, OutT *__restrict__ y, int32_t *__restrict__ acc_out, int M,
                      int N, int K) {
    using C = Cfg2;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[C::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // same offset in both CTAs

    const int tiles_m = (M + C::PM - 1) / C::PM;
    const int tiles_n = (N + C::BN - 1) / C::BN;
    const int num_tiles = tiles_m * tiles_n;
    const int num_kb = (K + BK - 1) / BK;
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tfull_bar[b]), 1);
            mbar_init(smem_u32(&tempty_bar[b]), 2 * kPairEpiWarps * 32);
        }
        mbar_init(smem_u32(&drain_bar), 1);
        abort_flag = 0;
        fence_barrier_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_a) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_b) : "memory");
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(&tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    pdl_wait();     // the codes and scales come from the previous kernel (prologue above overlapped it)
    pdl_trigger();  // the next kernel may launch; it waits for this grid before touching memory

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
                int tm, tn;
                tile_coords(tile, tiles_m, tiles_n, tm, tn);
                const int m0 = tm * C::PM + (int)rank * BM;
                const int n0 = tn * C::BN + (int)rank * (C::BN / 2);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, &abort_flag, kFaultProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_base + stage * C::STAGE_BYTES;
                    const uint32_t b_dst = a_dst + C::A_BYTES;
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    if (leader) mbar_arrive_expect_tx(fb, 2 * C::STAGE_BYTES);  // both CTAs' bytes
                    tma_load_2d_pair(a_dst, &tmap_a, fb & kPeerMask, kb * BK, m0);
                    tma_load_2d_pair(b_dst, &tmap_b, fb & kPeerMask, kb * BK, n0);
                    ++issued;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && leader) {
                // drain: wait (bounded) for the last issued stages to land
                int outstanding = issued < C::STAGES ? issued : C::STAGES;
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < outstanding; ++i) {
                    if (--s < 0) {
                        s = C::STAGES - 1;
                        ph ^= 1u;
                    }
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try_wait(smem_u32(&full_bar[s]), ph) && globaltimer() - t0 < kWaitNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader CTA only)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_i8(C::PM, C::BN);
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t buf_phase = 0;
            bool ok = true;
            bool issued_any = false;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
                if (!wait_bounded(smem_u32(&tempty_bar[buf]), buf_phase ^ 1u, &abort_flag, kFaultMmaTmemEmpty)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(buf * C::BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!wait_bounded(smem_u32(&full_bar[stage]), phase, &abort_flag, kFaultMmaFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_base + stage * C::STAGE_BYTES;
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        mma_i8_pair(d_tmem, smem_desc_sw128(a_addr + k * UMMA_K),
                                    smem_desc_sw128(b_addr + k * UMMA_K), idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    issued_any = true;
                    mma_commit_pair(smem_u32(&empty_bar[stage]));
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair(smem_u32(&tfull_bar[buf]));
                buf ^= 1;
                if (buf == 0) buf_phase ^= 1u;
            }
            if (!ok && issued_any) {
                mma_commit_pair(smem_u32(&drain_bar));
                const unsigned long long t0 = globaltimer();
                while (!mbar_try_wait(smem_u32(&drain_bar), 0) && globaltimer() - t0 < kWaitNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2.., both CTAs)
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int row_in_tile = (int)rank * BM + quarter * 32 + lane;
        constexpr int kCols = C::BN * 4 / kPairEpiWarps;   // columns of a tile per warp
        const int col0 = ((warp - 2) / 4) * kCols;
        const uint32_t out_buf = smem_base + C::OUT_OFFSET + (uint32_t)(warp - 2) * C::OUT_BYTES;
        bool store_pending = false;
        int buf = 0;
        uint32_t buf_phase = 0;
        for (int tile = pair; tile < num_tiles; tile += num_pairs) {
            int tm, tn;
            tile_coords(tile, tiles_m, tiles_n, tm, tn);
            const int m0 = tm * C::PM, n0 = tn * C::BN;
            const int row = m0 + row_in_tile;
            const float sxr = row < M ? sx[row] : 0.0f;
            const int Rr = (ASYM && row < M) ? rs[row] : 0;
            const bool ok = wait_bounded(smem_u32(&tfull_bar[buf]), buf_phase, &abort_flag, kFaultEpilogue);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * C::BN + col0);
            if (acc_out) {
                // with the int32 accumulators requested: direct stores of both
                epilogue_tile<OutT, ASYM>(tbase, row, M, n0 + col0, N, sxr, Rr, sw, ow, y, acc_out, kCols);
            } else {
                constexpr int CW = 128 / (int)sizeof(OutT);
#pragma unroll 1
                for (int c0 = 0; c0 < kCols; c0 += CW)
                    store_chunk_tma<OutT, ASYM>(&tmap_y, tbase + (uint32_t)c0, out_buf, lane, n0 + col0 + c0,
                                                m0 + (int)rank * BM + quarter * 32, M, N, sxr, Rr, sw, ow,
                                                store_pending);
            }
            tc_fence_before();
            mbar_arrive_leader(smem_u32(&tempty_bar[buf]));
            buf ^= 1;
            if (buf == 0) buf_phase ^= 1u;
        }
        if (lane == 0 && store_pending) bulk_wait_all();  // this warp's stores are complete
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the pair is done with TMEM and with each other's barriers
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// ============================================================ W4A8 kernel
// Weights as packed int4 (two codes per byte, element 2i in the low nibble,
// 4-bit two's complement).  Per stage TMA brings the A tile (int8, 128-byte
// swizzle) and the packed B tile (256 rows x 64 bytes, no swizzle); eight
// converter warps unpack B into int8 codes in the 128B-swizzled K-major layout
// the MMA reads (16-byte chunk c of row r at chunk c ^ (r & 7) of its
// 1024-byte row group), fence their writes to the async proxy and arrive on
// conv[s]; the MMA warp then runs the int8 MMAs of w8a8_gemm_kernel.  The
// weight bytes read from HBM are halved; the tensor-core work is the same.
constexpr int kConvWarps = 8;
constexpr int kThreadsW4 = (6 + kConvWarps) * 32;  // TMA, MMA, 4 epilogue and 8 converter warps

// Two rings: IN_STAGES input stages (A by TMA, 128-byte swizzle, and the
// packed B tile, 32 KB together) run ahead of OP_STAGES unpacked B buffers
// (32 KB each), so that loads from HBM do not wait on the conversion; the MMA
// reads A from the input stage and B from the operand buffer and releases
// both.
struct CfgW4 {
    static constexpr int BN = 256;
    static constexpr int IN_STAGES = 5;
    static constexpr int OP_STAGES = 2;
    static constexpr int A_BYTES = BM * BK;        // 16 KB int8 activations
    static constexpr int B_BYTES = BN * BK;        // 32 KB unpacked int8 weights
    static constexpr int RAW_BYTES = BN * BK / 2;  // 16 KB packed int4 weights
    static constexpr int IN_BYTES = A_BYTES + RAW_BYTES;
    static constexpr int IN_OFFSET = OP_STAGES * B_BYTES;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int SMEM = IN_OFFSET + IN_STAGES * IN_BYTES + 1024;
};


// 8 int4 codes (one 32-bit word, element 2i in the low nibble of byte i) to
// 8 int8 operands 16 q: a nibble moved to the high half of its byte, low
// half zero, is 16 times its signed value as an int8, so no sign extension
// is needed (|16 q| <= 128 stays in the int8 range).  The accumulator is then
// 16 times the product of the codes, exactly (every term is a multiple of
// 16, and |16 acc| < 2^31 for the sizes the GEMMs accept); the epilogues
// shift it right by 4 (exact) before the dequant.
constexpr int kInt4AccShift = 4;
__device__ __forceinline__ void unpack_int4x8(uint32_t w, uint32_t &o0, uint32_t &o1) {
    const uint32_t hi = w & 0xF0F0F0F0u;          // 16 q[2i+1]
    const uint32_t lo = (w << 4) & 0xF0F0F0F0u;   // 16 q[2i]
    o0 = __byte_perm(lo, hi, 0x5140);
    o1 = __byte_perm(lo, hi, 0x7362);
}

// Synchronisation (no block-level barrier in the main loop):
//   in_full[s]  : producer's expect_tx; the A and packed-B TMAs complete it.
//   in_empty[s] : MMA commit (the MMA is the last reader of A; the
//                 converters are done with the packed tile before op_full).
//   op_full[p]  : one arrival per converter thread after its fenced writes.
//   op_empty[p] : MMA commit.
template <typename OutT>
__global__ void __launch_bounds__(kThreadsW4, 1)
w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b4,
                 const float *__restrict__ sx, const float *__restrict__ sw, OutT *__restrict__ y,
                 int32_t *__restrict__ acc_out, int M, int N, int K) {
    using C = CfgW4;
    constexpr int BNw = C::BN;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t in_full[C::IN_STAGES];
    __shared__ __align__(8) uint64_t in_empty[C::IN_STAGES];
    __shared__ __align__(8) uint64_t op_full[C::OP_STAGES];
    __shared__ __align__(8) uint64_t op_empty[C::OP_STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // 1024-aligned for 128B swizzle
    uint8_t *gbase = smem_raw + (smem_base - smem_u32(smem_raw));      // the same bytes, generic address

    const int tiles_m = (M + BM - 1) / BM;
    const int tiles_n = (N + BNw - 1) / BNw;
    const int num_tiles = tiles_m * tiles_n;
    const int num_kb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::IN_STAGES; ++s) {
            mbar_init(smem_u32(&in_full[s]), 1);
            mbar_init(smem_u32(&in_empty[s]), 1);
        }
        for (int s = 0; s < C::OP_STAGES; ++s) {
            mbar_init(smem_u32(&op_full[s]), kConvWarps * 32);
            mbar_init(smem_u32(&op_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tfull_bar[b]), 1);
            mbar_init(smem_u32(&tempty_bar[b]), 4 * 32);
        }
        mbar_init(smem_u32(&drain_bar), 1);
        abort_flag = 0;
        fence_barrier_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_a) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmap_b4) : "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    pdl_wait();     // the codes and scales come from the previous kernel (prologue above overlapped it)
    pdl_trigger();  // the next kernel may launch; it waits for this grid before touching memory

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (A + packed B)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m0 = (tile % tiles_m) * BM, n0 = (tile / tiles_m) * BNw;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!wait_bounded(smem_u32(&in_empty[stage]), phase ^ 1u, &abort_flag, kFaultProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_base + C::IN_OFFSET + stage * C::IN_BYTES;
                    const uint32_t fb = smem_u32(&in_full[stage]);
                    mbar_arrive_expect_tx(fb, C::IN_BYTES);
                    tma_load_2d(a_dst, &tmap_a, fb, kb * BK, m0);
                    tma_load_2d(a_dst + C::A_BYTES, &tmap_b4, fb, kb * (BK / 2), n0);
                    ++issued;
                    if (++stage == C::IN_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                int outstanding = issued < C::IN_STAGES ? issued : C::IN_STAGES;
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < outstanding; ++i) {
                    if (--s < 0) {
                        s = C::IN_STAGES - 1;
                        ph ^= 1u;
                    }
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try_wait(smem_u32(&in_full[s]), ph) && globaltimer() - t0 < kWaitNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(BM, BNw);
            int stage = 0, istage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t buf_phase = 0;
            bool ok = true;
            bool issued_any = false;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!wait_bounded(smem_u32(&tempty_bar[buf]), buf_phase ^ 1u, &abort_flag, kFaultMmaTmemEmpty)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BNw);
                for (int kb = 0; kb < num_kb; ++kb) {
                    // op_full implies in_full: the converters waited for it
                    if (!wait_bounded(smem_u32(&op_full[stage]), phase, &abort_flag, kFaultMmaFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_base + C::IN_OFFSET + istage * C::IN_BYTES;
                    const uint32_t b_addr = smem_base + stage * C::B_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        mma_i8(d_tmem, smem_desc_sw128(a_addr + k * UMMA_K), smem_desc_sw128(b_addr + k * UMMA_K),
                               idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    issued_any = true;
                    mma_commit(smem_u32(&op_empty[stage]));
                    mma_commit(smem_u32(&in_empty[istage]));
                    if (++stage == C::OP_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++istage == C::IN_STAGES) istage = 0;
                }
                if (!ok) break;
                mma_commit(smem_u32(&tfull_bar[buf]));
                buf ^= 1;
                if (buf == 0) buf_phase ^= 1u;
            }
            if (!ok && issued_any) {
                mma_commit(smem_u32(&drain_bar));
                const unsigned long long t0 = globaltimer();
                while (!mbar_try_wait(smem_u32(&drain_bar), 0) && globaltimer() - t0 < kWaitNs) {
                }
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------ converters (warps 6..13)
        // Per k-block every converter thread waits for a free operand buffer
        // and for the input stage, unpacks its share of the packed tile into
        // the buffer, fences the writes to the async proxy and arrives on
        // op_full.
        const int cw = warp - 6;
        const int rsub = lane >> 2, sub = lane & 3;   // 8 rows x 4 lanes of 16 packed bytes per warp step
        int rs = 0, os = 0;
        uint32_t rph = 0, oph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!wait_bounded(smem_u32(&op_empty[os]), oph ^ 1u, &abort_flag, kFaultConvert)) {
                    ok = false;
                    break;
                }
                if (!wait_bounded(smem_u32(&in_full[rs]), rph, &abort_flag, kFaultConvert)) {
                    ok = false;
                    break;
                }
                const uint8_t *raw = gbase + C::IN_OFFSET + rs * C::IN_BYTES + C::A_BYTES;
                uint8_t *bdst = gbase + os * C::B_BYTES;
#pragma unroll 2
                for (int it = 0; it < BNw / (8 * kConvWarps); ++it) {
                    const int r = (it * kConvWarps + cw) * 8 + rsub;
                    const uint4 p = *reinterpret_cast<const uint4 *>(raw + r * (BK / 2) + sub * 16);
                    uint32_t o[8];
                    unpack_int4x8(p.x, o[0], o[1]);
                    unpack_int4x8(p.y, o[2], o[3]);
                    unpack_int4x8(p.z, o[4], o[5]);
                    unpack_int4x8(p.w, o[6], o[7]);
                    uint8_t *rowp = bdst + (r >> 3) * 1024 + (r & 7) * 128;
                    const int c0 = 2 * sub, c1 = 2 * sub + 1;
                    *reinterpret_cast<uint4 *>(rowp + ((c0 ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4 *>(rowp + ((c1 ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
                }
                fence_proxy_async_smem();  // the MMA reads these bytes through the async proxy
                mbar_arrive(smem_u32(&op_full[os]));
                if (++rs == C::IN_STAGES) {
                    rs = 0;
                    rph ^= 1u;
                }
                if (++os == C::OP_STAGES) {
                    os = 0;
                    oph ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        int buf = 0;
        uint32_t buf_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int m0 = (tile % tiles_m) * BM, n0 = (tile / tiles_m) * BNw;
            const int row = m0 + row_in_tile;
            const float sxr = row < M ? sx[row] : 0.0f;
            const bool ok = wait_bounded(smem_u32(&tfull_bar[buf]), buf_phase, &abort_flag, kFaultEpilogue);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BNw);
            epilogue_tile<OutT, false, kInt4AccShift>(tbase, row, M, n0, N, sxr, 0, sw, nullptr, y, acc_out, BNw);
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty_bar[buf]));
            buf ^= 1;
            if (buf == 0) buf_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace gemm
}  // namespace w8a8

#include "gemm_decode.cuh"

namespace w8a8 {
namespace gemm {

// Packs int8 codes in [-8, 7] two per byte (element 2i in the low nibble);
// one thread per 8 output bytes.
__global__ void pack_int4_kernel(const int8_t *__restrict__ q, int64_t total_out8, uint8_t *__restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total_out8;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 c = __ldg(reinterpret_cast<const uint4 *>(q) + i);  // 16 codes
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
        uint32_t p[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t v = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t word = w[2 * h + (b >> 1)];
                const uint32_t lo = (word >> (16 * (b & 1))) & 0xFu;
                const uint32_t hi = (word >> (16 * (b & 1) + 8)) & 0xFu;
                v |= (lo | (hi << 4)) << (8 * b);
            }
            p[h] = v;
        }
        reinterpret_cast<uint2 *>(out)[i] = make_uint2(p[0], p[1]);
    }
}

// One CTA waits, with the same bounded wait the GEMM uses, on an mbarrier
// that nothing ever arrives at: the wait must run out, record
// kFaultSelftest and return, leaving the context usable.
__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    wait_bounded(smem_u32(&bar), 0, &abort_flag, kFaultSelftest, limit_ns);
}

// ------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    }
    return fn;
}

// 2-D int8 tensor [rows, K] (K contiguous), box [box_rows, 128 bytes], 128B swizzle.
static bool make_map(CUtensorMap *map, const void *base, int64_t rows, int64_t K, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output y [rows, cols] (bf16 or fp32) for TMA stores: box [32 rows, 128
// bytes], 128B swizzle.  cols * element size is a multiple of 16 (checked by
// the entry points).
static bool make_map_out(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, bool bf16) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int64_t esz = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * esz)};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Packed int4 weights [rows, K/2 bytes]: box [box_rows, 64 bytes] (BK codes),
// no swizzle (the converter warps read it with plain loads).
// box_bytes packed bytes of each of box_rows rows; swizzle128: the 128-byte
// rows of a box land in shared memory with 16-byte piece j of row r at
// piece j ^ (r & 7) (TMA 128B swizzle)
static bool make_map_int4(CUtensorMap *map, const void *base, int64_t rows, int64_t K, int box_rows,
                          int box_bytes = BK / 2, bool swizzle128 = false) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename OutT>
static sq_status launch_w4(const int8_t *qx, const float *sx, const uint8_t *qw4, const float *sw, int M, int N,
                           int K, void *y, int32_t *acc_out, int sms, cudaStream_t st) {
    using C = CfgW4;
    CUtensorMap ma, mb;
    if (!make_map(&ma, qx, M, K, BM) || !make_map_int4(&mb, qw4, N, K, C::BN))
        return fail(SQ_ERR_CUDA, "w4a8_gemm_dequant: cuTensorMapEncodeTiled failed");
    auto kern = w4a8_gemm_kernel<OutT>;
    static int configured_dev[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured_dev[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        configured_dev[dev] = 1;
    }
    const int tiles = ((M + BM - 1) / BM) * ((N + C::BN - 1) / C::BN);
    const int grid = std::min(tiles, sms);
    launch_pdl(kern, dim3(grid), dim3(kThreadsW4), C::SMEM, st, ma, mb, sx, sw, (OutT *)y, acc_out, M, N, K);
    return launch_status("w4a8_gemm_kernel");
}

// K split of the decode kernel: the largest power of two S <= 8 with
// tiles x S CTAs <= two per SM and S <= k-blocks of kblock K each (every
// CTA gets one).
static int decode_split(int N, int K, int sms, int kblock) {
    const int tiles = (N + kDecRows - 1) / kDecRows;
    const int num_kb = (K + kblock - 1) / kblock;
    int s = 1;
    while (s < kDecMaxSplit && tiles * (2 * s) <= 2 * sms && 2 * s <= num_kb) s *= 2;
    return s;
}

template <int NT, typename OutT, bool ASYM, bool INT4>
static sq_status launch_decode(const int8_t *qx, const float *sx, const int32_t *rs, const void *qw,
                               const float *sw, const float *ow, int M, int N, int K, void *y, int32_t *acc_out,
                               int sms, cudaStream_t st) {
    using C = CfgDec<NT, INT4>;
    CUtensorMap mw, mx;
    const bool okw = INT4 ? make_map_int4(&mw, qw, N, K, kDecRows, C::KB / 2, true) : make_map(&mw, qw, N, K, kDecRows);
    if (!okw || !make_map(&mx, qx, M, K, NT))
        return fail(SQ_ERR_CUDA, "w8a8 decode GEMM: cuTensorMapEncodeTiled failed");
    auto kern = w8a8_gemm_decode_kernel<NT, OutT, ASYM, INT4>;
    static int configured_dev[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured_dev[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        // the whole shared-memory carveout, so that two CTAs fit an SM
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        configured_dev[dev] = 1;
    }
    const int split = decode_split(N, K, sms, C::KB);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(((N + kDecRows - 1) / kDecRows) * split), 1, 1);
    cfg.blockDim = dim3(dec_threads(INT4), 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mw, mx, sx, sw, rs, ow, (OutT *)y, acc_out, M, N, K);
    if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "w8a8_gemm_decode_kernel launch: %s", cudaGetErrorString(e));
    return launch_status("w8a8_gemm_decode_kernel");
}

// Token-tile width of the decode kernel: 16, 32 or 64 tokens, and 128 for
// int8 weights with 64 < M <= 128 (see gemm_entry).
template <typename OutT, bool ASYM, bool INT4>
static sq_status dispatch_decode(const int8_t *qx, const float *sx, const int32_t *rs, const void *qw,
                                 const float *sw, const float *ow, int M, int N, int K, void *y, int32_t *acc_out,
                                 int sms, cudaStream_t st) {
    if (M <= 16) return launch_decode<16, OutT, ASYM, INT4>(qx, sx, rs, qw, sw, ow, M, N, K, y, acc_out, sms, st);
    if (M <= 32) return launch_decode<32, OutT, ASYM, INT4>(qx, sx, rs, qw, sw, ow, M, N, K, y, acc_out, sms, st);
    if constexpr (!INT4) {
        if (M > 64) return launch_decode<128, OutT, ASYM, false>(qx, sx, rs, qw, sw, ow, M, N, K, y, acc_out, sms, st);
    }
    return launch_decode<64, OutT, ASYM, INT4>(qx, sx, rs, qw, sw, ow, M, N, K, y, acc_out, sms, st);
}

template <int BN, typename OutT, bool ASYM>
static sq_status launch(const int8_t *qx, const float *sx, const int32_t *rs, const int8_t *qw, const float *sw,
                        const float *ow, int M, int N, int K, void *y, int32_t *acc_out, int sms, cudaStream_t st) {
    using C = Cfg<BN>;
    CUtensorMap ma, mb;
    if (!make_map(&ma, qx, M, K, BM) || !make_map(&mb, qw, N, K, BN))
        return fail(SQ_ERR_CUDA, "w8a8_gemm_dequant: cuTensorMapEncodeTiled failed");
    auto kern = w8a8_gemm_kernel<BN, OutT, ASYM>;
    static int configured_dev[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured_dev[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        configured_dev[dev] = 1;
    }
    const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int grid = std::min(tiles, sms);
    launch_pdl(kern, dim3(grid), dim3(kThreads), C::SMEM, st, ma, mb, sx, sw, rs, ow, (OutT *)y, acc_out, M, N, K);
    return launch_status("w8a8_gemm_kernel");
}

template <typename OutT, bool ASYM>
static sq_status launch_pair(const int8_t *qx, const float *sx, const int32_t *rs, const int8_t *qw,
                             const float *sw, const float *ow, int M, int N, int K, void *y, int32_t *acc_out,
                             int sms, cudaStream_t st) {
    using C = Cfg2;
    CUtensorMap ma, mb, my;
    if (!make_map(&ma, qx, M, K, BM) || !make_map(&mb, qw, N, K, C::BN / 2) ||
        !make_map_out(&my, y, M, N, sizeof(OutT) == 2))
        return fail(SQ_ERR_CUDA, "w8a8_gemm_dequant: cuTensorMapEncodeTiled failed");
    auto kern = w8a8_gemm_pair_kernel<OutT, ASYM>;
    static int configured_dev[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured_dev[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        configured_dev[dev] = 1;
    }
    const int tiles = ((M + C::PM - 1) / C::PM) * ((N + C::BN - 1) / C::BN);
    const int pairs = std::min(tiles, sms / 2);
    launch_pdl(kern, dim3(2 * pairs), dim3(kThreadsPair), C::SMEM, st, ma, mb, my, sx, sw, rs, ow, (OutT *)y, acc_out,
               M, N, K);
    return launch_status("w8a8_gemm_pair_kernel");
}

}  // namespace gemm
}  // namespace w8a8

using namespace w8a8;

// Argument checks and dispatch shared by the symmetric and asymmetric
// entry points (rs/ow non-NULL: asymmetric weights).
static sq_status gemm_entry(const char *fn, const int8_t *qx, const float *sx, const int32_t *rs, const int8_t *qw,
                            const float *sw, const float *ow, int64_t M, int64_t N, int64_t K, void *y,
                            sq_dtype yt, int32_t *acc_out, void *stream) {
    const bool asym = rs != nullptr;
    if (M > 0 && N > 0 && (!qx || !sx || !qw || !sw || !y || (asym && !ow)))
        return fail(SQ_ERR_NULL, "%s: NULL pointer", fn);
    if (yt != SQ_F32 && yt != SQ_BF16) return fail(SQ_ERR_DTYPE, "%s: output dtype %d", fn, (int)yt);
    if (M < 0 || N < 0 || K <= 0 || K % 16 != 0 || K > (asym ? 65792 : 133144) || M > INT32_MAX || N > INT32_MAX)
        return fail(SQ_ERR_SHAPE, "%s: M=%lld N=%lld K=%lld (K a multiple of 16 in [16, %d])", fn, (long long)M,
                    (long long)N, (long long)K, asym ? 65792 : 133144);
    if (M == 0 || N == 0) return SQ_OK;
    const int out_vec = (yt == SQ_BF16) ? 8 : 4;
    if (N % out_vec != 0)
        return fail(SQ_ERR_SHAPE, "%s: N=%lld must be a multiple of %d for this output dtype", fn, (long long)N,
                    out_vec);
    if (acc_out && N % 4 != 0) return fail(SQ_ERR_SHAPE, "%s: acc_out needs N %% 4 == 0", fn);
    if (!aligned(qx, 16) || !aligned(qw, 16) || !aligned(y, 16) || !aligned(sw, 16) || !aligned(sx, 4) ||
        (acc_out && !aligned(acc_out, 16)) || (asym && (!aligned(ow, 16) || !aligned(rs, 4))))
        return fail(SQ_ERR_ALIGN, "%s: misaligned pointer (qx, qw, y, sw, ow, acc_out need 16 bytes)", fn);
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    const int m = (int)M, n = (int)N, k = (int)K;
    // M <= 64: the weight-streaming decode kernel; M > 128: 256-row tiles on
    // CTA pairs; otherwise one CTA per 128 x 256 tile, except where those
    // tiles would leave most SMs idle over a long K: the decode kernel with
    // 128-token tiles then splits K over a cluster (measured on B200 at 100
    // to 128 tokens: 128 x 4096 -> 4096 20.5 against 26.6 us, 100 x 133136
    // -> 16 74 against 372 us; with 43 column tiles, 128 x 4096 -> 11008, or
    // a short K the one-CTA kernel stays ahead: 28.7 against 34.8 us)
    const bool few_tiles = M <= 2 * gemm::kDecMaxTokens && (N + 255) / 256 <= sms / 8 && K >= 2048;
    if (M <= gemm::kDecMaxTokens || few_tiles) {
        if (yt == SQ_BF16)
            return asym ? gemm::dispatch_decode<__nv_bfloat16, true, false>(qx, sx, rs, qw, sw, ow, m, n, k, y,
                                                                            acc_out, sms, cs)
                        : gemm::dispatch_decode<__nv_bfloat16, false, false>(qx, sx, rs, qw, sw, ow, m, n, k, y,
                                                                             acc_out, sms, cs);
        return asym ? gemm::dispatch_decode<float, true, false>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs)
                    : gemm::dispatch_decode<float, false, false>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs);
    }
    if (M > gemm::BM) {
        if (yt == SQ_BF16)
            return asym ? gemm::launch_pair<__nv_bfloat16, true>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs)
                        : gemm::launch_pair<__nv_bfloat16, false>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs);
        return asym ? gemm::launch_pair<float, true>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs)
                    : gemm::launch_pair<float, false>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs);
    }
    if (yt == SQ_BF16)
        return asym ? gemm::launch<256, __nv_bfloat16, true>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs)
                    : gemm::launch<256, __nv_bfloat16, false>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs);
    return asym ? gemm::launch<256, float, true>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs)
                : gemm::launch<256, float, false>(qx, sx, rs, qw, sw, ow, m, n, k, y, acc_out, sms, cs);
}

extern "C" sq_status w8a8_gemm_dequant(const int8_t *qx, const float *sx, const int8_t *qw, const float *sw,
                                       int64_t M, int64_t N, int64_t K, void *y, sq_dtype yt, int32_t *acc_out,
                                       void *stream) {
    return gemm_entry("w8a8_gemm_dequant", qx, sx, nullptr, qw, sw, nullptr, M, N, K, y, yt, acc_out, stream);
}

extern "C" sq_status w8a8_gemm_dequant_asym(const int8_t *qx, const float *sx, const int32_t *rowsum,
                                            const int8_t *qw, const float *sw, const float *ow, int64_t M,
                                            int64_t N, int64_t K, void *y, sq_dtype yt, int32_t *acc_out,
                                            void *stream) {
    if (M > 0 && N > 0 && !rowsum) return fail(SQ_ERR_NULL, "w8a8_gemm_dequant_asym: NULL pointer");
    return gemm_entry("w8a8_gemm_dequant_asym", qx, sx, rowsum, qw, sw, ow, M, N, K, y, yt, acc_out, stream);
}

extern "C" sq_status w4a8_gemm_dequant(const int8_t *qx, const float *sx, const uint8_t *qw4, const float *sw,
                                       int64_t M, int64_t N, int64_t K, void *y, sq_dtype yt, int32_t *acc_out,
                                       void *stream) {
    const char *fn = "w4a8_gemm_dequant";
    if (M > 0 && N > 0 && (!qx || !sx || !qw4 || !sw || !y)) return fail(SQ_ERR_NULL, "%s: NULL pointer", fn);
    if (yt != SQ_F32 && yt != SQ_BF16) return fail(SQ_ERR_DTYPE, "%s: output dtype %d", fn, (int)yt);
    // the accumulator holds 16 acc (unpack_int4x8): 16 * 128 * 8 * K < 2^31
    if (M < 0 || N < 0 || K <= 0 || K % 32 != 0 || K > 131040 || M > INT32_MAX || N > INT32_MAX)
        return fail(SQ_ERR_SHAPE, "%s: M=%lld N=%lld K=%lld (K a multiple of 32 in [32, 131040])", fn, (long long)M,
                    (long long)N, (long long)K);
    if (M == 0 || N == 0) return SQ_OK;
    const int out_vec = (yt == SQ_BF16) ? 8 : 4;
    if (N % out_vec != 0)
        return fail(SQ_ERR_SHAPE, "%s: N=%lld must be a multiple of %d for this output dtype", fn, (long long)N,
                    out_vec);
    if (acc_out && N % 4 != 0) return fail(SQ_ERR_SHAPE, "%s: acc_out needs N %% 4 == 0", fn);
    if (!aligned(qx, 16) || !aligned(qw4, 16) || !aligned(y, 16) || !aligned(sw, 16) || !aligned(sx, 4) ||
        (acc_out && !aligned(acc_out, 16)))
        return fail(SQ_ERR_ALIGN, "%s: misaligned pointer (qx, qw4, y, sw, acc_out need 16 bytes)", fn);
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    if (M <= gemm::kDecMaxTokens) {
        if (yt == SQ_BF16)
            return gemm::dispatch_decode<__nv_bfloat16, false, true>(qx, sx, nullptr, qw4, sw, nullptr, (int)M,
                                                                     (int)N, (int)K, y, acc_out, sms, cs);
        return gemm::dispatch_decode<float, false, true>(qx, sx, nullptr, qw4, sw, nullptr, (int)M, (int)N, (int)K, y,
                                                         acc_out, sms, cs);
    }
    if (yt == SQ_BF16)
        return gemm::launch_w4<__nv_bfloat16>(qx, sx, qw4, sw, (int)M, (int)N, (int)K, y, acc_out, sms, cs);
    return gemm::launch_w4<float>(qx, sx, qw4, sw, (int)M, (int)N, (int)K, y, acc_out, sms, cs);
}

extern "C" sq_status sq_pack_int4(const int8_t *q, int64_t N, int64_t K, uint8_t *packed, void *stream) {
    if (N > 0 && (!q || !packed)) return fail(SQ_ERR_NULL, "sq_pack_int4: NULL pointer");
    if (N < 0 || K <= 0 || K % 32 != 0)
        return fail(SQ_ERR_SHAPE, "sq_pack_int4: N=%lld K=%lld (K a positive multiple of 32)", (long long)N,
                    (long long)K);
    if (N == 0) return SQ_OK;
    if (!aligned(q, 16) || !aligned(packed, 16)) return fail(SQ_ERR_ALIGN, "sq_pack_int4: misaligned pointer");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    const int64_t units = N * K / 16;
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(units, 256), 8LL * sms);
    gemm::pack_int4_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(q, units, packed);
    return launch_status("pack_int4_kernel");
}

extern "C" sq_status sq_selftest_bounded_wait(uint32_t limit_ms, void *stream) {
    if (limit_ms == 0 || limit_ms > 10000)
        return fail(SQ_ERR_ARG, "sq_selftest_bounded_wait: limit_ms=%u outside [1, 10000]", limit_ms);
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    gemm::bounded_wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)limit_ms * 1000000ull);
    return launch_status("bounded_wait_selftest_kernel");
}

extern "C" sq_status sq_device_fault(void *stream, uint32_t *fault_out) {
    if (!fault_out) return fail(SQ_ERR_NULL, "sq_device_fault: NULL pointer");
    cudaStream_t cs = (cudaStream_t)stream;
    unsigned int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_gemm_fault, sizeof v, 0, cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_gemm_fault, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "sq_device_fault: %s", cudaGetErrorString(e));
    *fault_out = v;
    return SQ_OK;
}
