// gemv_mma.cu -- the activation-sparse GEMV for batch 5..16, on the tensor cores.
//
//   y[b][n] = sum_{k in U} s[g(k)][n] * (q[k][n] - z[g(k)][n]) * x[b][k]
//
// U is the one active set of the batch (the union of the rows' active
// channels, found by the CTAs themselves from x and the rows' thresholds, or
// the caller's index list or bitmask). Method: "Enabling Dynamic
// Sparsity in Quantized LLM Inference", Abstract: a GEMV over the quantized
// layout that reads only the weight runs of the active channels.
//
// With B batch rows every weight code is used B times. The CUDA-core kernel
// (one FMA per code and batch row) is bound by FMA issue well before HBM from
// B of about 4, and above 8 rows each of its warps carries every row of its
// CTA; there each code is expanded once into an exact fp16 operand and the
// products go to the tensor cores (tcgen05.mma kind::f16, fp32 accumulators
// in tensor memory):
//  * Every CTA takes an equal share of the (tile, row) space, tiles of 1024
//    outputs (512 bytes of a packed row); a share that ends one tile and
//    starts the next is processed as two segments.
//  * The CTA's rows are cut into runs of one quantization group, and each run
//    into K-blocks of 32 rows (two MMA K-steps; 16 where two 64 KB operand
//    stages do not fit shared memory), a run's last block padded with zero
//    rows.
//  * 16 expanding warps; warp w expands slots w and w + 16 of every K-block.
//    Its lanes read their own 16-byte columns of its rows into registers (one
//    K-block ahead) and store each code as the exact fp16 value q 2^-24 (2^-20
//    for the high nibble of a byte): one AND per two codes, no zero point. A
//    K-block's A operand (1024 outputs x its rows, M-major, 128-byte swizzle)
//    and B operand (its rows x 16 batch columns of x' = x 2^S_b in fp16,
//    K-major) go to one of 2..4 stages.
//  * A 17th warp issues the K-block's MMAs (9 per K-step: M = 128 outputs,
//    N = 16, K = 16, the ninth with an all-ones A operand, so that its
//    accumulator holds the sum of x' over the run) into the run's accumulator
//    set (one of two, 9 x 16 columns of tensor memory each), then commits them
//    to the stage's "empty" barrier and, at a run's end, to the set's "ready"
//    barrier.
//  * One K-block into the next run the expanding warps read their outputs'
//    sums D and the row sums X from tensor memory and fold them with the
//    group's scale and zero into running totals, also in tensor memory:
//    total += s (2^c D - z X), i.e. the sum of s (q - z) x'. The products
//    are exact (fp16 x fp16), summed in fp32.
//  * Split-K partials go into the fp32 workspace with float reductions; the
//    shared epilogue kernel turns the workspace into bf16 y.
//
// Every wait on a barrier is bounded by 0.2 s of wall time; a wait that runs
// out sets SGQ_STATUS_TIMEOUT, the thread waits on nothing further and the
// kernel runs to its end (y is then not valid). Before the tensor memory is
// freed, the issuing thread waits (bounded too) for a commit that covers every
// MMA of the CTA; if that wait runs out as well, the memory is freed with MMAs
// possibly in flight (keeping it would leave the next allocation on the SM
// waiting for ever), so a timed-out call leaves that SM's tensor memory
// undefined until the stream drains. The kernel takes more than half of an SM's shared memory, so
// at most one of its CTAs is resident per SM and the allocation of all 512
// tensor-memory columns never waits.
#include "gemv_rows.cuh"
#include "sgq_device.cuh"
#include "sgq_launch.h"

#include <algorithm>
#include <type_traits>

namespace sgq {

namespace {

constexpr int kMWarps = 16;                 // warps that expand rows (one slot each) and fold
constexpr int kIssuer = kMWarps;            // one more warp issues the MMAs
constexpr int kAllWarps = kMWarps + 1;
constexpr int kMThreads = kAllWarps * 32;
constexpr int kKStep = 16;                  // the fp16 MMA's K
constexpr int kMmaN = 16;                   // MMA N: batch columns, padded to 16
constexpr int kMBlocks = kTileN1 / 128;     // MMA M-blocks per tile
// A K-block (one hand-off between the expanding warps and the issuer) holds
// KB = 16 or 32 rows: its A operand is KB x 1024 outputs (32 or 64 KB), its B
// operand KB x 16 batch columns; warp w expands slots w and w + 16.
__host__ __device__ constexpr int a_stage_bytes(int kb) { return kb * kTileN1 * 2; }
__host__ __device__ constexpr int b_stage_bytes(int kb) { return kb * kMmaN * 2; }
constexpr int kMaxStages = 4;               // operand stages (2..4, by shared memory)
constexpr int kPfRows = 2;                  // rows of packed codes in flight per expanding lane (one K-block)
constexpr int kTmemCols = 512;              // two accumulator sets and the running totals
// An accumulator set: the tile's 8 M-blocks and the row-sum block (below),
// 16 columns each, 160 columns apart; the totals after both sets.
constexpr int kSetCols = 160;
constexpr int kSumCol = kMBlocks * kMmaN;    // the row-sum block inside a set
constexpr int kTotCol = 2 * kSetCols;        // first column of the totals
constexpr int kOnesBytes = 4096;             // the all-ones A operand of the row-sum block
constexpr unsigned long long kWaitNs = 200000000ull; // a barrier wait gives up after 0.2 s
// A thread in a barrier wait sleeps until the phase completes or this many
// ns pass (then checks the wall-time limit), instead of spinning on it.
constexpr unsigned kSuspendNs = 20000;
constexpr size_t kOneCtaSmem = 116 * 1024;  // more than half of the SM's shared memory

static_assert(kSumCol + kMmaN <= kSetCols, "an accumulator set");
static_assert(kTotCol + kMBlocks * kMmaN <= kTmemCols, "accumulators and totals");

// Instruction descriptor of tcgen05.mma kind::f16: fp32 D, fp16 A and B,
// A M-major, B K-major, N = 16, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 15) | ((uint32_t)(kMmaN >> 3) << 17) |
                            ((uint32_t)(128 >> 4) << 24);

// Shared-memory matrix descriptor (sm_100 form): start, leading and stride
// byte offsets in 16-byte units, version 1, layout type (0 none, 2 128B swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) |
           ((uint64_t)(layout & 7u) << 61);
}

// Byte offset, inside a K-block's A stage, of the 16-byte chunk that lane l
// writes for word j of its 16-byte column of slot k. The stage is 16 atoms
// (64 outputs x 8 rows, 1 KB, 128-byte swizzle) along M times 2 along K. Lane
// l = 8g + h puts word j into atom g + 4j, logical chunk h, so that the 8
// lanes of each group g cover all 32 banks in every store.
__device__ __forceinline__ uint32_t a_chunk_off(int lane, int j, int k)
{
    const int g = lane >> 3, h = lane & 7, r = k & 7;
    return (uint32_t)((k >> 3) * (16 * 1024) + (g + 4 * j) * 1024 + r * 128 + ((h ^ r) << 4));
}

// Output (0..1023, within the tile) held by M slot m of the A operand: the
// inverse of the placement above. Chunk element e of word j carries output
// 8j + (e >> 1) + 4 (e & 1): an AND takes codes 8j + i and 8j + i + 4 into
// the two halves of a register.
__host__ __device__ constexpr int mma_out_of_slot(int m)
{
    return 32 * (8 * ((m >> 6) & 3) + ((m >> 3) & 7)) + 8 * (m >> 8) + ((m & 7) >> 1) +
           4 * (m & 1);
}

// Byte offset of element (batch column c, slot k) in a K-block's B stage:
// K-major, no swizzle, core matrices of 8 columns x 8 slots (16-byte rows),
// 128 bytes apart along K and KB / 8 x 128 along N.
__device__ __forceinline__ uint32_t b_elem_off(int c, int k, int kb)
{
    return (uint32_t)((k & 7) * 2 + (c & 7) * 16 + (k >> 3) * 128 + (c >> 3) * (kb / 8) * 128);
}

struct SmemM {
    size_t a, ones, b, rxh, ridx, rstart, rkb, kbt, scan, total;
};

__host__ __device__ inline size_t align16(size_t v) { return (v + 15) / 16 * 16; }

// Row stride of the staged x' (batch-major): an odd multiple of 8 rows, so
// that the 16 batch columns of one row fall into distinct bank pairs.
__host__ __device__ inline int rxh_stride(int rows_cap) { return (((rows_cap + 7) / 8) | 1) * 8; }

// a: `stages` A stages (1024-aligned); ones: the row-sum block's A operand
// (fp16 1.0, 1024-aligned); b: B stages; rxh: x' of the CTA's
// rows, [bp batch rows][stride] fp16; ridx: the CTA's rows; rstart / rkb:
// first row / first K-block of each run (+1 entry); kbt: per K-block, its
// first row and a word of its valid rows (bits 0-7), its run (bits 8-28),
// whether it opens its run (bit 30) and whether the previous run folds
// after it (bit 29); scan: per-32-row counts.
__host__ __device__ inline SmemM smemm_layout(int rows_cap, int stages, int bp, int kb)
{
    SmemM s;
    s.a = 0;
    s.ones = s.a + (size_t)stages * a_stage_bytes(kb);
    s.b = s.ones + kOnesBytes;
    s.rxh = s.b + (size_t)stages * b_stage_bytes(kb);
    s.ridx = align16(s.rxh + (size_t)bp * rxh_stride(rows_cap) * 2);
    s.rstart = align16(s.ridx + (size_t)rows_cap * 4);
    s.rkb = align16(s.rstart + (size_t)(rows_cap + 1) * 4);
    s.kbt = align16(s.rkb + (size_t)(rows_cap + 1) * 4);
    s.scan = align16(s.kbt + (size_t)(rows_cap + 1) * 8);
    s.total = align16(s.scan + (size_t)((rows_cap + 31) / 32 + 4) * 4);
    return s;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for the phase of the given parity to complete, for at most kWaitNs of
// wall time; a thread whose earlier wait gave up (ok == false) does not wait
// again, so that a broken hand-off ends the kernel within a fraction of a
// second. Returns ok.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, bool ok)
{
    if (!ok)
        return false;
    unsigned long long t0 = 0;
    for (;;) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done)
                     : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendNs)
                     : "memory");
        if (done)
            return true;
        const unsigned long long t = global_ns();
        if (t0 == 0)
            t0 = t;
        else if (t - t0 > kWaitNs)
            return false;
    }
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// One MMA; the descriptors come as their 32-bit halves, so that the issuer
// offsets a K-block's descriptors with one 32-bit add each (the start-address
// field never carries into the next field inside shared memory).
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint32_t alo, uint32_t ahi, uint32_t blo,
                                        uint32_t bhi, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t.reg .b64 a, b;\n\tsetp.ne.b32 p, %5, 0;\n\t"
                 "mov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %4};\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %6, p;\n\t}" ::"r"(d_tmem),
                 "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(accumulate), "r"(kIdesc)
                 : "memory");
}

// The completion of every MMA this thread issued so far arrives once on bar.
__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 16 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld16(uint32_t addr, float *d)
{
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,"
                 "%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(addr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int c = 0; c < 16; ++c)
        d[c] = __uint_as_float(r[c]);
}

__device__ __forceinline__ void tmem_st16(uint32_t addr, const float *v)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,"
                 "%11,%12,%13,%14,%15,%16};" ::"r"(addr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
                 "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
                 "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])),
                 "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
                 "r"(__float_as_uint(v[15]))
                 : "memory");
}

// A 16-byte shared-memory store at a compile-time offset from addr.
template <int OFF>
__device__ __forceinline__ void st_shared_v4_at(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                                uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0+%5], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b),
                 "r"(c), "r"(d), "n"(OFF)
                 : "memory");
}


// Rows of one segment into ridx (ascending positions of the caller's list, or
// of the active channels), returns their number. Index list: entries
// [lo, hi) of idx (outside [0, K) -> -1, flagged); dense: channels
// [8 lo, 8 hi); bitmask or threshold: the active channels of [8 lo, 8 hi)
// (mask bit, or |x[b][c]| > t_b for some batch row b), by ballots over runs of
// 32 channels and a prefix over the runs' counts. All threads; ends with a
// barrier.
template <int SRC>
__device__ int segment_rows(const GemvProblem &p, int lo, int hi, int32_t *ridx, int *scan,
                            uint16_t *rxh, int rs)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (SRC == ROWS_LIST) {
        for (int j = tid; j < hi - lo; j += kMThreads) {
            int k = __ldg(p.idx + lo + j);
            if ((unsigned)k >= (unsigned)p.K) {
                set_status(p.status, SGQ_STATUS_BAD_INDEX);
                k = -1;
            }
            ridx[j] = k;
        }
        __syncthreads();
        return hi - lo;
    } else if (SRC == ROWS_DENSE) {
        const int c0 = 8 * lo, n = 8 * (hi - lo);
        for (int j = tid; j < n; j += kMThreads)
            ridx[j] = c0 + j;
        __syncthreads();
        return n;
    } else {
        // bitmask: bit c of the mask; threshold: |x[b][c]| > t_b for some
        // batch row b (the union of the rows' active sets)
        const int c0 = 8 * lo, c1 = 8 * hi;
        const int runs = (c1 - c0 + 31) / 32;
        auto run_bits = [&](int q) -> uint32_t {
            const int c = c0 + q * 32 + lane;
            bool act = false;
            if (c < c1) {
                if (SRC == ROWS_MASK) {
                    act = (__ldg(p.mask + (c >> 5)) >> (c & 31)) & 1u;
                } else {
                    for (int b = 0; b < p.B; ++b)
                        act |= (fabsf(bf16_bits_to_float(__ldg(p.x + (size_t)b * p.K + c))) >
                                      p.tb[b]);
                }
            }
            return __ballot_sync(0xffffffffu, act);
        };
        for (int q = warp; q < runs; q += kAllWarps) {
            const uint32_t m = run_bits(q);
            if (lane == 0)
                scan[q] = __popc(m);
        }
        __syncthreads();
        int total = 0;
        for (int c = 0; c * 32 < runs; ++c) {
            int ct;
            const int excl = chunk_prefix(scan, runs, c, total, &ct);
            for (int q = c * 32 + ((warp - c * 32) % kAllWarps + kAllWarps) % kAllWarps;
                 q < runs && q < c * 32 + 32; q += kAllWarps) {
                const int base = __shfl_sync(0xffffffffu, excl, q - c * 32);
                if (SRC == ROWS_THRESH) {
                    // The same test, keeping the rows' x: an active channel's x
                    // goes to rxh (batch-major) at its position, so that the
                    // x' staging needs no second gather.
                    const int ch = c0 + q * 32 + lane;
                    uint16_t v[kMmaN];
                    bool act = false;
    #pragma unroll
                    for (int b = 0; b < kMmaN; ++b) {
                        v[b] = (b < p.B && ch < c1) ? __ldg(p.x + (size_t)b * p.K + ch) : (uint16_t)0;
                        act |= (b < p.B && ch < c1) &&
                               (fabsf(bf16_bits_to_float(v[b])) > p.tb[b]);
                    }
                    const uint32_t m = __ballot_sync(0xffffffffu, act);
                    if (act) {
                        const int j = base + __popc(m & ((1u << lane) - 1u));
                        ridx[j] = ch;
    #pragma unroll
                        for (int b = 0; b < kMmaN; ++b)
                            if (b < p.B)
                                rxh[(size_t)b * rs + j] = v[b];
                    }
                } else {
                    const uint32_t m = run_bits(q);
                    if ((m >> lane) & 1u)
                        ridx[base + __popc(m & ((1u << lane) - 1u))] = c0 + q * 32 + lane;
                }
            }
            total += ct;
        }
        __syncthreads();
        return total;
    }
}

template <int SRC, int KB>
__global__ void __launch_bounds__(kMThreads, 1) gemv_mma_kernel(const KParams kp)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bar_full[kMaxStages], bar_empty[kMaxStages];
    __shared__ __align__(8) uint64_t bar_ready[2], bar_free[2], bar_done;
    __shared__ uint32_t s_tmem;
    __shared__ int s_nruns, s_nkb;
    __shared__ int s_S[kMmaN];

    const GemvProblem &p = kp.p;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nst = kp.stages, bp = kp.bp;
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    constexpr int SPW = KB / 16; // slots per expanding warp
    constexpr int AST = a_stage_bytes(KB), BST = b_stage_bytes(KB);
    const SmemM L = smemm_layout(kp.rows_cap, nst, bp, KB);
    uint16_t *rxh = reinterpret_cast<uint16_t *>(smem + L.rxh);
    int32_t *ridx = reinterpret_cast<int32_t *>(smem + L.ridx);
    int *rstart = reinterpret_cast<int *>(smem + L.rstart);
    int *rkb = reinterpret_cast<int *>(smem + L.rkb);
    int2 *kbt = reinterpret_cast<int2 *>(smem + L.kbt);
    int *scan = reinterpret_cast<int *>(smem + L.scan);
    const uint32_t sA = smem_u32(smem + L.a), sB = smem_u32(smem + L.b);
    const uint32_t sOnes = smem_u32(smem + L.ones);

    // The row-sum block's A operand: every element fp16 1.0, so that its
    // accumulator holds, in every row, the sum of x' over the run's rows for
    // each batch column (whatever the operand's layout, all elements being
    // equal). Written once, made visible to the tensor core's reads.
    for (int i = tid; i < kOnesBytes / 16; i += kMThreads)
        reinterpret_cast<uint4 *>(smem + L.ones)[i] =
            make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
    // The B stages start at zero: batch columns past B are never written.
    for (int i = tid; i < nst * BST / 16; i += kMThreads)
        reinterpret_cast<uint4 *>(smem + L.b)[i] = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&s_tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(bar_full + s, kMWarps);
            mbar_init(bar_empty + s, 1);
        }
        for (int d = 0; d < 2; ++d) {
            mbar_init(bar_ready + d, 1);
            mbar_init(bar_free + d, kMWarps);
        }
        mbar_init(&bar_done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    grid_launch_dependents();
    const int lg = kp.lg;
    bool ok = true;

    // With a fixed row source (dense, bitmask, threshold) the channels of this
    // CTA's first segment are known now: their x (every batch row) is
    // requested into L2 before the wait, a hint only (the loads after the
    // wait see whatever the previous kernel wrote).
    if (SRC != ROWS_LIST && warp == 0 && lane < p.B) {
        const long long W0 = (long long)kp.n_tiles * (p.K / 8);
        const int v0 = (int)(W0 * blockIdx.x / gridDim.x), v1 = (int)(W0 * (blockIdx.x + 1) / gridDim.x);
        const int pt = p.K / 8, t0 = v0 / pt;
        const int lo = v0 - t0 * pt, hi = min(pt, v1 - t0 * pt);
        if (hi > lo)
            prefetch_l2_bulk(p.x + (size_t)lane * p.K + 8 * lo, 16u * (uint32_t)(hi - lo));
    }
    grid_dependency_wait(); // x, idx, count, mask may come from the previous kernel

    // This CTA's equal share [u0, u1) of the (tile, row) work: units of one
    // list entry (index list) or of 8 channels (dense, bitmask) per tile, so
    // that every SM gets the same amount whatever the number of tiles. A share
    // may end one tile and start the next: each part is a segment, processed
    // in turn, each adding into the workspace. Barrier phases and the
    // accumulator sets run on CTA-wide K-block and run counters.
    int per_tile;
    if (SRC == ROWS_LIST) {
        const int c = __ldg(p.count);
        per_tile = c < 0 ? 0 : (c > p.K ? p.K : c);
        if (per_tile != c && tid == 0 && blockIdx.x == 0)
            set_status(p.status, SGQ_STATUS_BAD_COUNT);
    } else {
        per_tile = p.K / 8;
    }
    const long long W = (long long)kp.n_tiles * per_tile; // < 2^31 (checked by the launcher)
    const int u0 = (int)(W * blockIdx.x / gridDim.x);
    const int u1 = (int)(W * (blockIdx.x + 1) / gridDim.x);
    int kb_base = 0, run_base = 0;
    for (int u = u0; u < u1;) {
        const int tile = u / per_tile;
        const int lo = u - tile * per_tile;
        const int hi = min(per_tile, u1 - tile * per_tile);
        u = tile * per_tile + hi;
        const int n0 = tile * kTileN1;
        const int nvalid_out = min(kTileN1, p.N - n0); // outputs of this tile
        const bool lane_ok = 32 * lane < nvalid_out;
        __syncthreads(); // the previous segment's readers of the row arrays are done

        // The segment's rows (invalid list entries are -1: read as row 0, x = 0).
        const int nr = segment_rows<SRC>(p, lo, hi, ridx, scan, rxh, rxh_stride(kp.rows_cap));
        auto grp = [&](int j) { return max(ridx[j], 0) >> lg; };

        // Runs of one group: starts by ballots over chunks of 32 rows, positions
        // by a prefix over the chunks' counts.
        const int chunks = (nr + 31) / 32;
        for (int q = warp; q < chunks; q += kAllWarps) {
            const int j = q * 32 + lane;
            const bool st = (j < nr) && (j == 0 || grp(j) != grp(j - 1));
            const uint32_t m = __ballot_sync(0xffffffffu, st);
            if (lane == 0)
                scan[q] = __popc(m);
        }
        __syncthreads();
        {
            int total = 0;
            for (int c = 0; c * 32 < chunks; ++c) {
                int ct;
                const int excl = chunk_prefix(scan, chunks, c, total, &ct);
                for (int q = c * 32 + ((warp - c * 32) % kAllWarps + kAllWarps) % kAllWarps;
                     q < chunks && q < c * 32 + 32; q += kAllWarps) {
                    const int base = __shfl_sync(0xffffffffu, excl, q - c * 32);
                    const int j = q * 32 + lane;
                    const bool st = (j < nr) && (j == 0 || grp(j) != grp(j - 1));
                    const uint32_t m = __ballot_sync(0xffffffffu, st);
                    if (st)
                        rstart[base + __popc(m & ((1u << lane) - 1u))] = j;
                }
                total += ct;
            }
            if (tid == 0) {
                s_nruns = total;
                rstart[total] = nr;
            }
        }
        __syncthreads();
        const int nruns = s_nruns;
        // First K-block of each run: a prefix over the runs' K-block counts.
        if (warp == 0) {
            int carry = 0;
            for (int c = 0; c * 32 < nruns; ++c) {
                const int r = c * 32 + lane;
                const int v = (r < nruns) ? (rstart[r + 1] - rstart[r] + KB - 1) / KB : 0;
                int incl = v;
    #pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d)
                        incl += t;
                }
                if (r < nruns)
                    rkb[r] = carry + incl - v;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) {
                rkb[nruns] = carry;
                s_nkb = carry;
            }
        }
        __syncthreads();
        const int nkb = s_nkb;
        // First row, valid rows, run and flags of every K-block (its run by a
        // binary search over the runs' first K-blocks), so that the expansion
        // warps read one word per K-block instead of walking the runs. The
        // previous run folds one K-block into a run (on its only K-block when
        // it has one). rows_cap, bounded by shared memory, keeps the run index
        // far inside its 21 bits.
        for (int t = tid; t < nkb; t += kMThreads) {
            int lo = 0, hi = nruns - 1; // the run r with rkb[r] <= t < rkb[r + 1]
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (rkb[mid] <= t)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            const int j0 = rstart[lo] + KB * (t - rkb[lo]);
            const int fkb = rkb[lo] + min(1, rkb[lo + 1] - rkb[lo] - 1);
            kbt[t] = make_int2(j0, min(rstart[lo + 1] - j0, KB) | (lo << 8) |
                                       ((t == rkb[lo]) << 30) | ((t == fkb) << 29));
        }
        __syncthreads();

        // The issuer's run of K-block kb (a pointer advanced monotonically).
        auto kb_run = [&](int kb, int &run) {
            while (kb >= rkb[run + 1])
                ++run;
        };

        if (warp == kIssuer) {
            // ---- the MMA issuer --------------------------------------------------
            if (lane == 0) {
                int run = 0;
                int ist = kb_base % nst, iph = (kb_base / nst) & 1; // stage, phase of K-block 0
                const uint64_t od = smem_desc(sOnes, 1024, 2048, 2);
                for (int kb = 0; kb < nkb; ++kb) {
                    kb_run(kb, run);
                    const bool first = kb == rkb[run], last = kb == rkb[run + 1] - 1;
                    const int rg = run_base + run;
                    const int s = ist;
                    ok = mbar_wait(bar_full + s, (uint32_t)iph, ok);
                    if (++ist == nst) {
                        ist = 0;
                        iph ^= 1;
                    }
                    tc_fence_after();
                    if (first && rg >= 2) {
                        ok = mbar_wait(bar_free + (rg & 1), (uint32_t)(((rg >> 1) - 1) & 1), ok);
                        tc_fence_after();
                    }
                    const uint32_t dcol = tmem + (uint32_t)(kSetCols * (rg & 1));
                    const uint64_t ad = smem_desc(sA + (uint32_t)(s * AST), 1024, 16 * 1024, 2);
                    const uint64_t bd = smem_desc(sB + (uint32_t)(s * BST), 128, (KB / 8) * 128, 0);
                    const uint32_t alo = (uint32_t)ad, ahi = (uint32_t)(ad >> 32);
                    const uint32_t blo = (uint32_t)bd, bhi = (uint32_t)(bd >> 32);
                    // Every M-block: a lane's outputs are spread over the M-blocks
                    // (lanes past N hold finite codes of column 0 and are dropped
                    // in the epilogue); then the row sums of x'.
    #pragma unroll
                    for (int kk = 0; kk < KB / kKStep; ++kk) {
                        const uint32_t acc = (kk > 0 || !first) ? 1u : 0u;
                        const uint32_t bk = blo + (uint32_t)((kk * 256) >> 4);
    #pragma unroll
                        for (int mb = 0; mb < kMBlocks; ++mb)
                            mma_f16(dcol + (uint32_t)(kMmaN * mb),
                                    alo + (uint32_t)((kk * 32768 + mb * 2048) >> 4), ahi, bk, bhi,
                                    acc);
                        mma_f16(dcol + (uint32_t)kSumCol, (uint32_t)od, (uint32_t)(od >> 32), bk,
                                bhi, acc);
                    }
                    mma_commit(bar_empty + s);
                    if (last && !(p.debug_withhold_ready && run == nruns - 1))
                        mma_commit(bar_ready + (rg & 1));
                }
            }
            __syncwarp();
        } else {
            // ---- the expanding warps ---------------------------------------------
            // Warp w expands slots w (and w + 16) of every K-block. Its lanes read
            // their 16-byte columns of those rows straight into registers,
            // kPfRows rows ahead, so that no shared memory carries packed codes.
            constexpr int kEx = kMWarps * 32; // threads of the expanding warps
            constexpr int PF = kPfRows / SPW; // K-blocks prefetched ahead
            // x' = x 2^S_b in fp16 per batch row b, 2^14 <= max |x'| < 2^15 over
            // the CTA's rows (as in the batch-1 kernel), staged batch-major in
            // rxh. Warp w owns batch row b = w: lane l gathers rows l, l + 32,
            // ... (one bf16 each, 32 loads in flight; consecutive channels make
            // each warp load one coalesced 64-byte request), then the warp
            // reduces max |x| and converts its row in place, 8 rows per lane
            // loaded before any is stored.
            const int rs = rxh_stride(kp.rows_cap);
            if (warp < p.B) {
                const int b = warp;
                uint16_t *xr = rxh + (size_t)b * rs;
                const uint16_t *xb = p.x + (size_t)b * p.K;
                float m = 0.f;
                if (SRC == ROWS_THRESH) { // the row selection staged x already
                    for (int j0 = 0; j0 < nr; j0 += 32 * 8) {
                        uint16_t v[8];
    #pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int j = j0 + 32 * u + lane;
                            v[u] = (j < nr) ? xr[j] : (uint16_t)0;
                        }
    #pragma unroll
                        for (int u = 0; u < 8; ++u)
                            m = fmaxf(m, fabsf(bf16_bits_to_float(v[u])));
                    }
                }
                for (int j0 = 0; SRC != ROWS_THRESH && j0 < nr; j0 += 32 * 32) {
                    uint16_t v[32];
    #pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const int j = j0 + 32 * u + lane;
                        const int k = (j < nr) ? ridx[j] : -1;
                        v[u] = (k >= 0) ? __ldg(xb + k) : (uint16_t)0;
                    }
    #pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const int j = j0 + 32 * u + lane;
                        if (j < nr) {
                            xr[j] = v[u];
                            m = fmaxf(m, fabsf(bf16_bits_to_float(v[u])));
                        }
                    }
                }
                const int e = warp_max_exponent(m);
                const int S = (e == INT32_MIN) ? 0 : 14 - e;
                if (lane == 0)
                    s_S[b] = S;
                const float fa = pow2f(S - S / 2), fb = pow2f(S / 2);
                __syncwarp();
                for (int j0 = 0; j0 < nr; j0 += 32 * 8) {
                    uint16_t v[8];
    #pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = j0 + 32 * u + lane;
                        v[u] = (j < nr) ? xr[j] : (uint16_t)0;
                    }
    #pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = j0 + 32 * u + lane;
                        if (j < nr)
                            xr[j] = __half_as_ushort(__float2half_rn((bf16_bits_to_float(v[u]) * fa) * fb));
                    }
                }
            }

            const size_t row_bytes = (size_t)(p.N / 2);
            const uint8_t *wcol = p.qweight + (lane_ok ? ((size_t)n0 / 2 + lane * 16) : 0);
            // This warp's rows of K-block kb into dst (zero for slots past the
            // K-block's valid rows; lanes past N read column 0).
            auto fetch = [&](int kb, uint4 *dst) {
                if (kb < nkb) {
                    const int2 e = kbt[kb];
                    const int j0 = e.x, nv = e.y & 0xFF;
    #pragma unroll
                    for (int u = 0; u < SPW; ++u) {
                        const int slot = warp + 16 * u;
                        dst[u] = make_uint4(0u, 0u, 0u, 0u);
                        if (slot < nv) {
                            const uint8_t *src =
                                wcol + (size_t)max(ridx[j0 + slot], 0) * row_bytes;
                            asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(dst[u].x), "=r"(dst[u].y), "=r"(dst[u].z),
                                           "=r"(dst[u].w)
                                         : "l"(src));
                        }
                    }
                }
            };
            uint4 pf[PF][SPW];
    #pragma unroll
            for (int q = 0; q < PF; ++q)
                fetch(q, pf[q]);
            // This lane's A chunks (stage-relative): word j of slot warp + 16 u
            // sits 4096 j + 32768 u bytes after that of word 0 of slot `warp`
            // (atoms g + 4 j, and two 8-row atom groups per 16 slots). Its B
            // element: warp b < B writes batch column b, lane l slot l.
            const uint32_t aoff = a_chunk_off(lane, 0, warp);
            const uint32_t boffc = b_elem_off(warp & (kMmaN - 1), lane & (KB - 1), KB);

            // Fold outputs of this thread: its tensor-memory lane (quadrant
            // warp % 4) in M-blocks 2 (warp / 4) and 2 (warp / 4) + 1.
            const int mbA = 2 * (warp >> 2);
            const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
            int fout[2];
    #pragma unroll
            for (int i = 0; i < 2; ++i)
                fout[i] = mma_out_of_slot(128 * (mbA + i) + 32 * (warp & 3) + lane);
            // (s, z) words of the fold outputs for a group, kept raw until the fold
            // so that the loads stay in flight.
            uint32_t sfold[2], snew[2];
            auto load_s = [&](int G, uint32_t *sv) {
    #pragma unroll
                for (int i = 0; i < 2; ++i)
                    sv[i] = (fout[i] < nvalid_out) ? __ldg(p.sz + (size_t)G * p.N + n0 + fout[i]) : 0u;
            };
            if (nruns > 0)
                load_s(grp(rstart[0]), snew);

            // totals += s (2^c D - z X) for run r's accumulators (set r & 1):
            // D sums the raw codes q 2^-c times x' over the run's rows, X (the
            // row-sum block) sums x', so that s (q - z) x' is summed with no
            // zero point in the operand (z: an integer-valued fp16, s z exact
            // in fp32). The totals stay in tensor memory (columns kTotCol..),
            // written by run 0.
            auto fold = [&](int r) { // r: run of this segment
                const int rg = run_base + r;
                ok = mbar_wait(bar_ready + (rg & 1), (uint32_t)((rg >> 1) & 1), ok);
                tc_fence_after();
                const uint32_t set = tmem + tlane + (uint32_t)(kSetCols * (rg & 1));
    #pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float d[kMmaN], t[kMmaN];
                    const float sc = __half2float(__ushort_as_half((uint16_t)(sfold[i] & 0xffffu)));
                    const float f = sc * ((fout[i] & 1) ? 1048576.f : 16777216.f);
                    const float nsz = -sc * __half2float(__ushort_as_half((uint16_t)(sfold[i] >> 16)));
                    tmem_ld16(set + kSumCol, d); // X
                    if (r == 0) {
    #pragma unroll
                        for (int c = 0; c < kMmaN; ++c)
                            t[c] = nsz * d[c];
                    } else {
                        tmem_ld16(tmem + tlane + kTotCol + kMmaN * (mbA + i), t);
    #pragma unroll
                        for (int c = 0; c < kMmaN; ++c)
                            t[c] = fmaf(nsz, d[c], t[c]);
                    }
                    tmem_ld16(set + kMmaN * (mbA + i), d); // D
    #pragma unroll
                    for (int c = 0; c < kMmaN; ++c)
                        t[c] = fmaf(f, d[c], t[c]);
                    tmem_st16(tmem + tlane + kTotCol + kMmaN * (mbA + i), t);
                }
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar_free + (rg & 1));
            };

            // every batch row's x' (written by its warp above) is in place
            asm volatile("bar.sync 1, %0;" ::"n"(kEx) : "memory");

            // K-block kb from the registers in v: expand into stage kb % nst,
            // the B operand beside it, hand the stage to the issuer; then the
            // previous run's fold, one K-block into the next run (its MMAs have
            // had that long to finish).
            int run = 0;
            int est = kb_base % nst, eph = (kb_base / nst) & 1; // stage, phase of K-block 0
            auto step = [&](int kb, const uint4 *v) {
                const int2 e = kbt[kb];
                const int fl = e.y, j0 = e.x;
                const int nv = fl & 0xFF; // valid slots of the K-block (at most KB)
                run = (fl >> 8) & 0x1FFFFF;
                const int kg = kb_base + kb;
                const int s = est;
                if (((fl >> 30) & 1) && run > 0) { // a run's first K-block
    #pragma unroll
                    for (int i = 0; i < 2; ++i)
                        sfold[i] = snew[i];
                    load_s(grp(rstart[run]), snew); // this run's (s, z), for its fold
                }
                // The stage's previous K-block has been multiplied.
                if (kg >= nst)
                    ok = mbar_wait(bar_empty + s, (uint32_t)(eph ^ 1), ok);
                const uint32_t a_st = sA + (uint32_t)(s * AST);
    #pragma unroll
                for (int u = 0; u < SPW; ++u) {
                    const uint32_t wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    // The raw codes as exact fp16 subnormals: q 2^-24 (low
                    // nibbles) and q 2^-20 (high); invalid slots hold zero
                    // codes and meet a zero B operand.
                    const uint32_t ab = a_st + aoff + 32768u * u;
                    auto put = [&](const uint32_t w, auto off) {
                        const uint32_t w8 = w >> 8;
                        st_shared_v4_at<decltype(off)::value>(ab, w & 0x000F000Fu, w & 0x00F000F0u,
                                                              w8 & 0x000F000Fu, w8 & 0x00F000F0u);
                    };
                    put(wv[0], std::integral_constant<int, 0>{});
                    put(wv[1], std::integral_constant<int, 4096>{});
                    put(wv[2], std::integral_constant<int, 8192>{});
                    put(wv[3], std::integral_constant<int, 12288>{});
                }
                if (warp < p.B && lane < KB) {
                    // B operand: x' of batch column `warp` for slot `lane` (zero
                    // past the K-block's valid rows), one coalesced read.
                    const uint16_t xv = (lane < nv) ? rxh[(size_t)warp * rs + j0 + lane] : (uint16_t)0;
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(sB + (uint32_t)(s * BST) + boffc),
                                 "h"(xv)
                                 : "memory");
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar_full + s);
                if (run > 0 && ((fl >> 29) & 1))
                    fold(run - 1);
                if (++est == nst) {
                    est = 0;
                    eph ^= 1;
                }
            };

            for (int kb0 = 0; kb0 < nkb; kb0 += PF) {
    #pragma unroll
                for (int q = 0; q < PF; ++q) {
                    const int kb = kb0 + q;
                    if (kb < nkb) {
                        step(kb, pf[q]);
                        fetch(kb + PF, pf[q]);
                    }
                }
            }
            if (nruns > 0) {
    #pragma unroll
                for (int i = 0; i < 2; ++i)
                    sfold[i] = snew[i];
                fold(nruns - 1);
            }
            // Split-K partials from the totals, back in real units (x 2^-S_b,
            // two exact factors).
            if (nkb > 0) {
                tc_fence_after();
    #pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float t[kMmaN];
                    tmem_ld16(tmem + tlane + kTotCol + kMmaN * (mbA + i), t);
                    if (fout[i] < nvalid_out) {
    #pragma unroll
                        for (int c = 0; c < kMmaN; ++c) {
                            if (c < p.B) {
                                const int E = -s_S[c];
                                atomicAdd(p.ws_acc + (size_t)c * p.N + n0 + fout[i],
                                          (t[c] * pow2f(E / 2)) * pow2f(E - E / 2));
                            }
                        }
                    }
                }
            }
        }
        kb_base += nkb;
        run_base += nruns;
    }
    if (warp == kIssuer && lane == 0) {
        // every MMA of this CTA has completed when bar_done's phase 0 does
        // (the tensor memory is freed only after that, below)
        mma_commit(&bar_done);
        ok = mbar_wait(&bar_done, 0u, true) && ok;
    }
    if (!ok)
        set_status(p.status, SGQ_STATUS_TIMEOUT);

    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
}

// Batch columns of the staged x: B rounded up to 2, 4, 8 or 16.
int pad_batch(int B)
{
    int b = 2;
    while (b < B)
        b *= 2;
    return b;
}

template <int SRC>
cudaError_t launch_mma_t(KParams kp, int num_sms, cudaStream_t stream)
{
    const GemvProblem &p = kp.p;
    kp.nb = 1;
    kp.bp = pad_batch(p.B);
    kp.n_tiles = ceil_div(p.N, kTileN1);
    kp.k_splits = 1; // unused: the grid shares the (tile, row) space evenly
    kp.span_cap = 0;
    // Each CTA an equal share of n_tiles x K/8 units of 8 rows; a segment
    // holds at most one share's rows. When a whole number of shares per tile
    // fills at least 90% of the SMs, shares stay inside tiles (a CTA that
    // spans two tiles pays the prologue and the tail twice, and the slowest
    // CTA sets the time); otherwise one share per SM. More CTAs (waves) only
    // if a share's rows do not fit shared memory.
    const long long units = (long long)kp.n_tiles * (p.K / 8);
    if ((long long)kp.n_tiles * p.K >= (1ll << 31))
        return cudaErrorInvalidValue; // the kernel's work units are 32-bit
    int grid = num_sms;
    if (kp.n_tiles <= num_sms && 10 * kp.n_tiles * (num_sms / kp.n_tiles) >= 9 * num_sms)
        grid = kp.n_tiles * (num_sms / kp.n_tiles);
    // 32-row K-blocks (half the hand-offs) when two stages of them fit with
    // the share's rows; else 16-row K-blocks, more CTAs only if even those do
    // not fit.
    for (const int kb : {32, 16}) {
        for (int g = grid;; g *= 2) {
            KParams kq = kp;
            kq.rows_cap = (int)(8 * ((units + g - 1) / g + 1) + 8);
            kq.rows_cap = std::min(kq.rows_cap, p.K + 8);
            kq.stages = kMaxStages;
            SmemM L = smemm_layout(kq.rows_cap, kq.stages, kq.bp, kb);
            while (kq.stages > 2 && L.total + 1024 > kMaxSmem) {
                --kq.stages;
                L = smemm_layout(kq.rows_cap, kq.stages, kq.bp, kb);
            }
            if (L.total + 1024 <= kMaxSmem) {
                const size_t smem = std::max(L.total + 1024, kOneCtaSmem);
                cudaError_t err =
                    (kb == 32) ? launch_pdl(gemv_mma_kernel<SRC, 32>, g, kMThreads, smem, stream, kq)
                               : launch_pdl(gemv_mma_kernel<SRC, 16>, g, kMThreads, smem, stream, kq);
                if (err != cudaSuccess || p.accumulate)
                    return err;
                return launch_finalize(p, stream);
            }
            if (kb == 32 || (long long)g >= units)
                break; // 32-row blocks only without extra waves
        }
    }
    return cudaErrorInvalidConfiguration;
}

} // namespace

cudaError_t launch_gemv_mma(const GemvProblem &p, int num_sms, cudaStream_t stream)
{
    KParams kp{};
    kp.p = p;
    kp.lg = __builtin_ctz((unsigned)p.group);
    switch (p.source) {
    case ROWS_LIST: return launch_mma_t<ROWS_LIST>(kp, num_sms, stream);
    case ROWS_DENSE: return launch_mma_t<ROWS_DENSE>(kp, num_sms, stream);
    case ROWS_MASK: return launch_mma_t<ROWS_MASK>(kp, num_sms, stream);
    case ROWS_THRESH: return launch_mma_t<ROWS_THRESH>(kp, num_sms, stream);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace sgq
