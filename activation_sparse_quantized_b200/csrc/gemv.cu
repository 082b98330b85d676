// gemv.cu -- the activation-sparse GEMV over group-wise int4 weights.
//
//   y[b][n] = sum_{k in S} s[g(k)][n] * (q[k][n] - z[g(k)][n]) * x[b][k]
//
// Method: "Enabling Dynamic Sparsity in Quantized LLM Inference", Abstract: a
// GEMV that works on the quantized layout and reads only the weights of the
// active input channels, gathered at run time. Layout version 1 keeps each
// channel's codes as one contiguous run (N/2 bytes), so an inactive channel
// costs no memory traffic at all.
//
// The path is HBM-bound (batch 1..16, no dense contraction, no tensor cores),
// and at these sizes the whole GEMV is about one latency-bandwidth product of
// HBM, so the kernel's job is to have nearly all of its bytes in flight early
// and to keep the arithmetic under the memory time:
//  * Outputs are cut into tiles of 1024 (512 bytes of a packed row); the rows
//    (active channels) of each tile into k_splits shares so that
//    n_tiles * k_splits CTAs cover the SMs.
//  * Scale/zero of the CTA's groups are prefetched first; in the threshold
//    path (select fused into the prologue) their span is known from the CTA's
//    channel slice, before x is read.
//  * Each warp takes a contiguous slice of the CTA's rows; every lane streams
//    its own 16-byte column of each row through a per-lane ring in shared
//    memory with cp.async, 8 rows ahead. A lane reads back only bytes it
//    copied itself: no barrier, only its own groups.
//  * Codes are summed per group without dequantizing
//    (sum s (q - z) x = s (sum q x - z sum x)). One 32-bit AND takes two codes
//    into the two halves of an fp16 pair, where they read as exact fp16
//    subnormals; a mixed-precision FMA (fp16 x fp16 + fp32) multiplies each by
//    x held in fp16 under a per-warp power-of-two scale, so every product is
//    exact. Scale and zero are applied once per (group, output) in a fold.
//  * B = 2..4: each warp carries two batch rows, which share the extracted codes;
//    the warps form ceil(B / 2) (rounded to a power of two) batch groups that
//    read the same rows, the later reads hitting L2, so HBM still sees each
//    active row once.
//  * Split-K: each warp leaves its partial tile in its own (drained) ring
//    region; after one barrier the CTA sums the warps' tiles (no shared
//    atomics: many-way float atomics on the same addresses serialize) and adds
//    the result into an fp32 workspace with vector reductions, then exits. A
//    second tiny kernel, chained with programmatic dependent launch, turns the
//    workspace into bf16 y and re-zeroes it once the GEMV grid has completed.
//  * Programmatic dependent launch: a GEMV lets the next kernel in the stream
//    launch early and itself waits for the previous one before it reads x,
//    idx or count or writes anything; only the packed weights are read before.
#include "gemv_rows.cuh"
#include "sgq_device.cuh"
#include "sgq_launch.h"

#include <algorithm>

namespace sgq {

namespace {

// Split-K epilogue, a second (tiny) kernel launched right behind the GEMV with
// programmatic dependent launch: it waits until the GEMV grid has completed
// (so every partial sum has been added into the workspace), converts the fp32
// sums to bf16 y, writes the optional fp32 copy and re-zeroes the workspace.
// Doing this in a kernel of its own keeps memory fences and tickets out of the
// GEMV's CTAs, which just add their partials and exit.
//
// GLU epilogues (the gated FFN fused behind one GEMV over the stacked gate
// and up weights): output i of row b is act(gate) * up with gate = sum[b][i]
// and up = sum[b][I + i], I = N / 2, computed from the fp32 sums and rounded
// once to bf16.
template <int EPI>
__global__ void __launch_bounds__(256) finalize_kernel(GemvProblem p)
{
    grid_launch_dependents();
    grid_dependency_wait();
    const int width = (EPI == EPI_PLAIN) ? p.N : p.N / 2; // outputs per row
    const int quads = width / 4;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < p.B * quads;
         e += gridDim.x * blockDim.x) {
        const int b = e / quads, i = (e % quads) * 4;
        float *wp = p.ws_acc + (size_t)b * p.N + i;
        float4 v = ld_cg_v4(wp);
        st_cg_v4(wp, make_float4(0.f, 0.f, 0.f, 0.f));
        if (EPI != EPI_PLAIN) {
            float *wu = wp + width;
            const float4 u = ld_cg_v4(wu);
            st_cg_v4(wu, make_float4(0.f, 0.f, 0.f, 0.f));
            constexpr int ACT = (EPI == EPI_GLU_SILU) ? SGQ_ACT_SILU : SGQ_ACT_RELU;
            v = make_float4(act_mul<ACT>(v.x, u.x), act_mul<ACT>(v.y, u.y),
                            act_mul<ACT>(v.z, u.z), act_mul<ACT>(v.w, u.w));
        }
        const size_t o = (size_t)b * width + i;
        uint2 yb;
        yb.x = (uint32_t)float_to_bf16_bits(v.x) | ((uint32_t)float_to_bf16_bits(v.y) << 16);
        yb.y = (uint32_t)float_to_bf16_bits(v.z) | ((uint32_t)float_to_bf16_bits(v.w) << 16);
        *reinterpret_cast<uint2 *>(p.y + o) = yb;
        if (p.y_f32)
            *reinterpret_cast<float4 *>(p.y_f32 + o) = v;
    }
    // sums consumed by this GEMV's prologue (the gate/up sums of a fused FFN)
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < p.zero_extra_n / 4;
         e += gridDim.x * blockDim.x)
        st_cg_v4(p.zero_extra + 4 * e, make_float4(0.f, 0.f, 0.f, 0.f));
}

// ---------------------------------------------------------------------------
// The GEMV kernel, 1 <= B <= 16
// ---------------------------------------------------------------------------

constexpr int kWarps1 = 8;
constexpr int kThreads1 = kWarps1 * 32;
constexpr int kStages1 = 8; // rows in flight per warp (power of two); deeper rings measured slower

// Batch rows per warp: 1 for B = 1, 2 for B > 1 (the codes a lane extracts
// from a row serve both). With B > 1 the warps form kp.nb batch groups of
// kWarps1 / nb warps; each group covers BW batch rows and reads the same rows
// as the other groups (the later reads hit L2).
__host__ __device__ constexpr int warp_region_bytes(int bw, bool nm = false)
{
    // a warp's ring, which also holds its partial tiles (BW x the tile's
    // outputs as floats: 1024, or 2048 for the 2:4 layout)
    return (kStages1 * kRowBytes1 > bw * kTileN1 * (nm ? 2 : 1) * 4)
               ? kStages1 * kRowBytes1
               : bw * kTileN1 * (nm ? 2 : 1) * 4;
}

// Output o (0..31) of a lane is code o % 8 of packed word o / 8. One 32-bit AND
// takes two codes of a word at once, one into each fp16 half: the masked half
// reads as the fp16 subnormal q * 2^-24 (codes 0, 2, 4, 6 of the word, the
// latter two after word >> 8) or q * 2^-20 (codes 1, 3, 5, 7, taken from bits
// 4..7 of the half). A mixed-precision FMA (fp16 operands, fp32 accumulator)
// multiplies it by x' in fp16: the product is exact and normal in fp32.
__host__ __device__ constexpr int code_shift(int o)
{
    return (o & 1) ? 20 : 24; // accumulator of output o holds sum q x' 2^-code_shift
}

struct Smem1 {
    size_t ring, szs, rxh, ridx, rx, scan, xs, total;
};

// ring: each warp's region (its kStages1 rows of 512 B, then its partial
// tiles). szs: the (s, z) fp16 pairs of the staged groups, 1024 words per
// group, lane l's 8 chunks of 4 words swizzled as part_chunk(l, c). ridx: the
// CTA's rows (channels). rx: x of each row, per batch row b at b * rows_cap.
// rxh: x' = x 2^S of each row as fp16, same indexing. xs: x of the CTA's
// channel slice (bitmask rows, batch 1). bp = batch rows padded to nb * BW.
__host__ __device__ inline Smem1 smem1_layout(int span_cap, int rows_cap, int bp, int bw,
                                              bool nm = false)
{
    Smem1 s;
    s.ring = 0;
    s.szs = s.ring + (size_t)kWarps1 * warp_region_bytes(bw, nm);
    s.ridx = s.szs + (size_t)span_cap * kTileN1 * 4;
    s.rx = s.ridx + (size_t)rows_cap * 4;
    s.scan = s.rx + (size_t)rows_cap * bp * 4;
    s.rxh = s.scan + (size_t)((rows_cap + 31) / 32 + 4) * 4;
    s.xs = s.rxh + ((size_t)rows_cap * bp * 2 + 15) / 16 * 16;
    s.total = s.xs + (size_t)rows_cap * 4;
    return s;
}

// One packed word (codes of outputs 8t .. 8t + 7 of the lane) times x' into
// a[0..7]: word >> 8 by mul.hi on the FMA pipe, four ANDs on the logic pipe,
// eight mixed-precision FMAs.
__device__ __forceinline__ void mac_word(uint32_t w, uint16_t xh, float *a)
{
    asm("{\n\t"
        ".reg .b32 h, p;\n\t"
        ".reg .f16 lo, hi;\n\t"
        "mul.hi.u32 h, %8, 16777216;\n\t"
        "and.b32 p, %8, 0x000F000F;\n\t"
        "mov.b32 {lo, hi}, p;\n\t"
        "fma.rn.f32.f16 %0, lo, %9, %0;\n\t"
        "fma.rn.f32.f16 %4, hi, %9, %4;\n\t"
        "and.b32 p, %8, 0x00F000F0;\n\t"
        "mov.b32 {lo, hi}, p;\n\t"
        "fma.rn.f32.f16 %1, lo, %9, %1;\n\t"
        "fma.rn.f32.f16 %5, hi, %9, %5;\n\t"
        "and.b32 p, h, 0x000F000F;\n\t"
        "mov.b32 {lo, hi}, p;\n\t"
        "fma.rn.f32.f16 %2, lo, %9, %2;\n\t"
        "fma.rn.f32.f16 %6, hi, %9, %6;\n\t"
        "and.b32 p, h, 0x00F000F0;\n\t"
        "mov.b32 {lo, hi}, p;\n\t"
        "fma.rn.f32.f16 %3, lo, %9, %3;\n\t"
        "fma.rn.f32.f16 %7, hi, %9, %7;\n\t"
        "}"
        : "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3]), "+f"(a[4]), "+f"(a[5]), "+f"(a[6]),
          "+f"(a[7])
        : "r"(w), "h"(xh));
}

// The same for two batch rows: one extraction, sixteen FMAs.
__device__ __forceinline__ void mac_word2(uint32_t w, uint16_t x0, uint16_t x1, float *a,
                                          float *b)
{
    asm("{\n\t"
        ".reg .b32 h, p;\n\t"
        ".reg .f16 lo, hi;\n\t"
        "mul.hi.u32 h, %16, 16777216;\n\t"
        "and.b32 p, %16, 0x000F000F;\n\t"
        "mov.b32 {lo, hi}, p;\n\t"
        "fma.rn.f32.f16 %0, lo, %17, %0;\n\t"
        "fma.rn.f32.f16 %4, hi, %17, %4;\n\t"
        "fma.rn.f32.f16 %8, lo, %18, %8;\n\t"
        "fma.rn.f32.f16 %12, hi, %18, %12;\n\t"
        "and.b32 p, %16, 0x00F000F0;\n\t"
        "mov.b32 {lo, hi}, p;\n\t"
        "fma.rn.f32.f16 %1, lo, %17, %1;\n\t"
        "fma.rn.f32.f16 %5, hi, %17, %5;\n\t"
        "fma.rn.f32.f16 %9, lo, %18, %9;\n\t"
        "fma.rn.f32.f16 %13, hi, %18, %13;\n\t"
        "and.b32 p, h, 0x000F000F;\n\t"
        "mov.b32 {lo, hi}, p;\n\t"
        "fma.rn.f32.f16 %2, lo, %17, %2;\n\t"
        "fma.rn.f32.f16 %6, hi, %17, %6;\n\t"
        "fma.rn.f32.f16 %10, lo, %18, %10;\n\t"
        "fma.rn.f32.f16 %14, hi, %18, %14;\n\t"
        "and.b32 p, h, 0x00F000F0;\n\t"
        "mov.b32 {lo, hi}, p;\n\t"
        "fma.rn.f32.f16 %3, lo, %17, %3;\n\t"
        "fma.rn.f32.f16 %7, hi, %17, %7;\n\t"
        "fma.rn.f32.f16 %11, lo, %18, %11;\n\t"
        "fma.rn.f32.f16 %15, hi, %18, %15;\n\t"
        "}"
        : "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3]), "+f"(a[4]), "+f"(a[5]), "+f"(a[6]),
          "+f"(a[7]), "+f"(b[0]), "+f"(b[1]), "+f"(b[2]), "+f"(b[3]), "+f"(b[4]), "+f"(b[5]),
          "+f"(b[6]), "+f"(b[7])
        : "r"(w), "h"(x0), "h"(x1));
}

// One row (16 bytes = 4 words of this lane) into the group accumulators of
// the warp's BW batch rows.
template <int BW>
__device__ __forceinline__ void mac_row(const uint4 &v, const uint16_t *xh, float (*accg)[32])
{
    if (BW == 1) {
        mac_word(v.x, xh[0], accg[0]);
        mac_word(v.y, xh[0], accg[0] + 8);
        mac_word(v.z, xh[0], accg[0] + 16);
        mac_word(v.w, xh[0], accg[0] + 24);
    } else {
        mac_word2(v.x, xh[0], xh[1], accg[0], accg[BW - 1]);
        mac_word2(v.y, xh[0], xh[1], accg[0] + 8, accg[BW - 1] + 8);
        mac_word2(v.z, xh[0], xh[1], accg[0] + 16, accg[BW - 1] + 16);
        mac_word2(v.w, xh[0], xh[1], accg[0] + 24, accg[BW - 1] + 24);
    }
}

__device__ __forceinline__ float half_lo(uint32_t w)
{
    return __half2float(__ushort_as_half((uint16_t)(w & 0xffffu)));
}

__device__ __forceinline__ float half_hi(uint32_t w)
{
    return __half2float(__ushort_as_half((uint16_t)(w >> 16)));
}

// Float4 slot of outputs 32l + 4c .. 32l + 4c + 3 (lane l, chunk c) inside a
// warp's partial tile: the chunk index is XOR-ed with l & 7 so that a warp's
// 128-bit stores (fixed c) and the readers' 128-bit loads (fixed l) are free
// of bank conflicts.
__device__ __forceinline__ int part_chunk(int l, int c)
{
    return 8 * l + (c ^ (l & 7));
}

// The same for the 2:4 layout's 64 outputs per lane (16 chunks of 4).
__device__ __forceinline__ int part_chunk16(int l, int c)
{
    return 16 * l + (c ^ (l & 15));
}

// NM: the 2:4 layout (batch 1): the codes of a row are the kept outputs'
// slots, 1024 slots = 2048 outputs per tile, 64 outputs per lane; the fold
// adds each slot's sum to its output through the group's keep nibbles.
// SEG (index list, or the batch-row threshold): instead of (tile, split) from
// the block index, the CTA takes an equal share of the (tile, list entry)
// space, or of the (tile, 8-channel unit) space, which may end one tile and
// start the next; each part (segment) runs the whole body in turn, adding into
// the workspace.
template <int SRC, int BW, bool NM = false, bool SEG = false>
__global__ void __launch_bounds__(kThreads1, 1) gemv_kernel(const KParams kp)
{
    static_assert(!NM || BW == 1, "the 2:4 layout is batch 1 only");
    constexpr int OPL = NM ? 64 : 32;  // outputs per lane
    constexpr int TO = 32 * OPL;       // outputs per tile
    extern __shared__ __align__(16) uint8_t smem[];
    const GemvProblem &p = kp.p;
    const int bp = kp.nb * BW; // batch rows padded to whole groups
    const Smem1 L = smem1_layout(kp.span_cap, kp.rows_cap, bp, BW, NM);
    uint8_t *ring = smem + L.ring;
    const uint4 *szs = reinterpret_cast<const uint4 *>(smem + L.szs);
    int32_t *ridx = reinterpret_cast<int32_t *>(smem + L.ridx);
    float *rx = reinterpret_cast<float *>(smem + L.rx);
    uint16_t *rxh = reinterpret_cast<uint16_t *>(smem + L.rxh);
    int *scan = reinterpret_cast<int *>(smem + L.scan);
    const int rcap = kp.rows_cap;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // (tile, split), or with SEG the CTA's share of the list over the tiles
    int su = 0, su1 = 1, per_tile = 1;
    if constexpr (SEG) {
        grid_launch_dependents();
        if constexpr (SRC == ROWS_LIST) {
            grid_dependency_wait(); // x, idx, count may come from the previous kernel
            const int c = __ldg(p.count);
            per_tile = c < 0 ? 0 : (c > p.K ? p.K : c);
            if (per_tile != c && tid == 0 && blockIdx.x == 0)
                set_status(p.status, SGQ_STATUS_BAD_COUNT);
        } else {
            per_tile = p.K / 8; // channel units
        }
        const long long W = (long long)kp.n_tiles * per_tile;
        su = (int)(W * blockIdx.x / gridDim.x);
        su1 = (int)(W * (blockIdx.x + 1) / gridDim.x);
    }
    while (su < su1) {
        int tile, split = 0, seg_lo = 0, seg_hi = 0;
        if constexpr (SEG) {
            tile = su / per_tile;
            seg_lo = su - tile * per_tile;
            seg_hi = min(per_tile, su1 - tile * per_tile);
            su = tile * per_tile + seg_hi;
            __syncthreads(); // the previous segment is done with shared memory
        } else {
            tile = blockIdx.x % kp.n_tiles;
            split = blockIdx.x / kp.n_tiles;
            su = su1;
        }
        (void)seg_lo;
        (void)seg_hi;
        const int n0 = tile * TO;           // first output of the tile
        const int s0 = tile * kTileN1;      // first code slot of the tile
        const int SN = NM ? p.N / 2 : p.N;  // code slots (and (s, z) pairs) per row and group
        const int lg = kp.lg;
        const size_t row_stride = (size_t)(SN / 2);
        const bool lane_ok = (n0 + lane * OPL) < p.N;

        if constexpr (!SEG)
            grid_launch_dependents();

        // Scale/zero of the CTA's groups, staged asynchronously (the oldest
        // cp.async group of every thread). With a fixed channel slice (threshold /
        // mask / dense) the groups are known now, so the copies start before
        // waiting on the previous kernel; with an index list they follow the list.
        int G0 = 0, span = 0;
        auto stage_sz = [&]() {
            for (int c = tid; c < span * (kTileN1 / 4); c += kThreads1) {
                const int g = c >> 8, q = c & 255; // q: chunk of 4 slots in the tile
                if (s0 + 4 * q < SN)
                    cp_async16(smem + L.szs + ((size_t)g * 256 + part_chunk(q >> 3, q & 7)) * 16,
                               p.sz + (size_t)(G0 + g) * SN + s0 + 4 * q);
            }
            cp_async_commit();
        };
        if (SRC != ROWS_LIST) {
            int c0, c1;
            if (SEG) {
                c0 = 8 * seg_lo; // the segment's channel units (threshold source)
                c1 = 8 * seg_hi;
            } else if (SRC == ROWS_THRESH || SRC == ROWS_MASK || SRC == ROWS_GLU) {
                channel_slice(kp, split, c0, c1);
            } else {
                c0 = (int)((long long)p.K * split / kp.k_splits);
                c1 = (int)((long long)p.K * (split + 1) / kp.k_splits);
            }
            if (c1 > c0) {
                G0 = c0 >> lg;
                span = min(((c1 - 1) >> lg) - G0 + 1, kp.span_cap);
                // The slice of the input this CTA reads right after the wait
                // (x of each batch row, the gate/up sums, or the mask words),
                // requested into L2 now: a hint only, the loads after the wait
                // still see whatever the previous kernel wrote.
                if (warp == 0) {
                    if (SRC == ROWS_THRESH && lane < p.B)
                        prefetch_l2_bulk(p.x + (size_t)lane * p.K + c0, 2u * (uint32_t)(c1 - c0));
                    if (SRC == ROWS_GLU && lane < 2)
                        prefetch_l2_bulk(p.gu + (size_t)lane * p.K + c0, 4u * (uint32_t)(c1 - c0));
                    if (SRC == ROWS_MASK)
                        prefetch_l2_lines(p.mask + (c0 >> 5), p.mask + ((c1 - 1) >> 5) + 1);
                }
            }
            stage_sz();
        }

        if constexpr (!SEG || SRC != ROWS_LIST)
            grid_dependency_wait(); // x, idx, count, mask may come from the previous kernel

        // Rows (build_rows ends with a barrier). Invalid list entries stay -1: they
        // are read as row 0 with x = 0, so they add nothing.
        const int nr = build_rows<SRC, kThreads1, (BW == 1)>(
            kp, split, ridx, rx, scan, reinterpret_cast<float *>(smem + L.xs), tile == 0,
            SEG ? seg_lo : -1, SEG ? seg_hi : -1);
        auto row = [&](int j) { return (SRC == ROWS_LIST) ? max(ridx[j], 0) : ridx[j]; };

        if (SRC == ROWS_LIST) {
            if (nr > 0) {
                const int kf = row(0), kl = row(nr - 1);
                G0 = kf >> lg;
                span = min(max((kl >> lg) - G0 + 1, 1), kp.span_cap);
            }
            stage_sz(); // stays the oldest cp.async group
        }

        // This warp's batch rows and its contiguous slice of the CTA's rows.
        const int wpg = (BW == 1) ? kWarps1 : kWarps1 / kp.nb;
        const int b0 = (BW == 1) ? 0 : (warp / wpg) * BW;
        const int wq = (BW == 1) ? warp : warp % wpg;
        const int nbw = (BW == 1) ? 1 : max(0, min(BW, p.B - b0)); // real batch rows of this warp
        const int wa = (int)((long long)nr * wq / wpg);
        const int n = (nbw > 0) ? (int)((long long)nr * (wq + 1) / wpg) - wa : 0;

        // Ring prologue. Lanes past N read column 0 (valid memory, result unused).
        const uint8_t *wcol = p.qweight + (lane_ok ? ((size_t)s0 / 2 + lane * 16) : 0);
        uint8_t *region = ring + (size_t)warp * warp_region_bytes(BW, NM);
        uint8_t *myring = region + lane * 16;
    #pragma unroll
        for (int s = 0; s < kStages1; ++s) {
            if (s < n)
                cp_async16(myring + s * kRowBytes1, wcol + (size_t)row(wa + s) * row_stride);
            cp_async_commit();
        }

        // x of this warp's rows and batch rows (after the weights are in flight),
        // unless build_rows already read it (threshold; bitmask at batch 1).
        // Padded batch rows and invalid list entries get x = 0.
        if (!((SRC == ROWS_THRESH && BW == 1) || SRC == ROWS_GLU || (SRC == ROWS_MASK && BW == 1))) {
            for (int e = lane; e < n * BW; e += 32) {
                const int j = e / BW, bb = e - j * BW;
                const int k = ridx[wa + j];
                rx[(b0 + bb) * rcap + wa + j] =
                    (k >= 0 && bb < nbw) ? bf16_bits_to_float(__ldg(p.x + (size_t)(b0 + bb) * p.K + k))
                                         : 0.f;
            }
            __syncwarp();
        }

        // Per batch row: x' = x 2^S in fp16 with 2^14 <= max |x'| < 2^15 over the
        // warp's rows: exact for every |x| >= 2^-28 max |x| (fp16 normals);
        // smaller x round on the fp16 subnormal grid, an error below
        // 2^-39 max |x'|. Each product q 2^-24 x' (or q 2^-20 x') is then exact in
        // fp32.
        int S[BW];
    #pragma unroll
        for (int bb = 0; bb < BW; ++bb) {
            const float *xr = rx + (b0 + bb) * rcap;
            uint16_t *hr = rxh + (b0 + bb) * rcap;
            float m = 0.f;
            for (int j = lane; j < n; j += 32)
                m = fmaxf(m, fabsf(xr[wa + j]));
            const int e = warp_max_exponent(m);
            S[bb] = (e == INT32_MIN) ? 0 : 14 - e;
            const float fa = pow2f(S[bb] - S[bb] / 2), fb = pow2f(S[bb] / 2);
            for (int j = lane; j < n; j += 32)
                hr[wa + j] = __half_as_ushort(__float2half_rn((xr[wa + j] * fa) * fb));
        }
        __syncwarp();
        // The staged scale/zero (every thread's oldest cp.async group) have landed
        // and are visible to every warp before the first fold.
        cp_async_wait<kStages1>();
        __syncthreads();

        // accg[bb][o] = this group's sum of q x' 2^-code_shift(o) for code slot o;
        // acc[bb][o] = folded result of output o in units of 2^-S.
        float accg[BW][32], acc[BW][OPL];
    #pragma unroll
        for (int bb = 0; bb < BW; ++bb) {
    #pragma unroll
            for (int o = 0; o < 32; ++o)
                accg[bb][o] = 0.f;
    #pragma unroll
            for (int o = 0; o < OPL; ++o)
                acc[bb][o] = 0.f;
        }

        //   acc += s * (2^code_shift accg - z * sum x')
        auto fold = [&](int G, const float *Xg) {
            const bool staged = (G >= G0) && (G < G0 + span);
            uint32_t w[32]; // (s, z) of this lane's 32 outputs
            if (staged) {
    #pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = szs[(G - G0) * 256 + part_chunk(lane, c)];
                    w[4 * c] = v.x;
                    w[4 * c + 1] = v.y;
                    w[4 * c + 2] = v.z;
                    w[4 * c + 3] = v.w;
                }
            } else {
                const uint4 *g4 = reinterpret_cast<const uint4 *>(
                    p.sz + (size_t)G * SN + s0 + (lane_ok ? lane * 32 : 0));
    #pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = __ldg(g4 + c);
                    w[4 * c] = v.x;
                    w[4 * c + 1] = v.y;
                    w[4 * c + 2] = v.z;
                    w[4 * c + 3] = v.w;
                }
            }
            if (!NM) {
    #pragma unroll
                for (int o = 0; o < 32; ++o) {
                    const float s = half_lo(w[o]), z = half_hi(w[o]);
    #pragma unroll
                    for (int bb = 0; bb < BW; ++bb) {
                        const float t = accg[bb][o] * pow2f(code_shift(o));
                        acc[bb][o] = fmaf(s, fmaf(-z, Xg[bb], t), acc[bb][o]);
                        accg[bb][o] = 0.f;
                    }
                }
            } else {
                // Keep nibbles of this lane's 16 blocks (8 bytes); block j's slots
                // 2j, 2j + 1 go to its first and second kept output.
                const uint2 km = lane_ok ? __ldg(reinterpret_cast<const uint2 *>(
                                               p.keep + (size_t)G * (p.N / 8) + n0 / 8 + lane * 8))
                                         : make_uint2(0u, 0u);
    #pragma unroll
                for (int j = 0; j < 16; ++j) {
                    float f[2];
    #pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int o = 2 * j + h;
                        const float t = accg[0][o] * pow2f(code_shift(o));
                        f[h] = half_lo(w[o]) * fmaf(-half_hi(w[o]), Xg[0], t);
                        accg[0][o] = 0.f;
                    }
                    const uint32_t m = ((j < 8 ? km.x : km.y) >> (4 * (j & 7))) & 0xFu;
    #pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const bool kept = (m >> i) & 1u;
                        const bool second = (m & ((1u << i) - 1u)) != 0u; // a kept output below i
                        acc[0][4 * j + i] += kept ? (second ? f[1] : f[0]) : 0.f;
                    }
                }
            }
        };

        auto xrow = [&](int j, uint16_t *xh) {
    #pragma unroll
            for (int bb = 0; bb < BW; ++bb)
                xh[bb] = rxh[(b0 + bb) * rcap + wa + j];
        };

        // Runs of rows of one group: the run end comes from one ballot per 32
        // rows, and sum x' of the run from one warp reduction, so the per-row work
        // is the ring read, the codes and the refill only.
        int i = 0;
        while (i < n) {
            const int G = row(wa + i) >> lg;
            int i1 = i;
            float Xg[BW];
    #pragma unroll
            for (int bb = 0; bb < BW; ++bb)
                Xg[bb] = 0.f;
            for (;;) {
                const int j = i1 + lane;
                const bool in = (j < n) && ((row(wa + j) >> lg) == G);
                const uint32_t bal = __ballot_sync(0xffffffffu, in);
                const int len = (bal == 0xffffffffu) ? 32 : (__ffs(~bal) - 1);
                if (lane < len) {
    #pragma unroll
                    for (int bb = 0; bb < BW; ++bb)
                        Xg[bb] += __half2float(__ushort_as_half(rxh[(b0 + bb) * rcap + wa + j]));
                }
                i1 += len;
                if (len < 32)
                    break;
            }
    #pragma unroll
            for (int bb = 0; bb < BW; ++bb)
    #pragma unroll
                for (int d = 16; d > 0; d >>= 1)
                    Xg[bb] += __shfl_xor_sync(0xffffffffu, Xg[bb], d);

            for (; i + 1 < i1; i += 2) {
                cp_async_wait<kStages1 - 2>(); // rows i and i + 1 have landed
                const int slot = i & (kStages1 - 1), slot1 = (i + 1) & (kStages1 - 1);
                const uint4 v0 = *reinterpret_cast<const uint4 *>(myring + slot * kRowBytes1);
                const uint4 v1 = *reinterpret_cast<const uint4 *>(myring + slot1 * kRowBytes1);
                uint16_t xh0[BW], xh1[BW];
                xrow(i, xh0);
                xrow(i + 1, xh1);
                mac_row<BW>(v0, xh0, accg);
                mac_row<BW>(v1, xh1, accg);
                if (i + kStages1 < n)
                    cp_async16(myring + slot * kRowBytes1,
                               wcol + (size_t)row(wa + i + kStages1) * row_stride);
                cp_async_commit();
                if (i + 1 + kStages1 < n)
                    cp_async16(myring + slot1 * kRowBytes1,
                               wcol + (size_t)row(wa + i + 1 + kStages1) * row_stride);
                cp_async_commit();
            }
            if (i < i1) {
                // The last row of an odd-length run.
                cp_async_wait<kStages1 - 1>();
                const int slot = i & (kStages1 - 1);
                const uint4 v = *reinterpret_cast<const uint4 *>(myring + slot * kRowBytes1);
                uint16_t xh[BW];
                xrow(i, xh);
                mac_row<BW>(v, xh, accg);
                if (i + kStages1 < n)
                    cp_async16(myring + slot * kRowBytes1,
                               wcol + (size_t)row(wa + i + kStages1) * row_stride);
                cp_async_commit();
                ++i;
            }
            fold(G, Xg);
        }

        // This warp's partial tiles, in real units (x 2^-S, two exact factors),
        // into its own region: every cp.async of this warp has landed and been
        // read, so nothing else touches that region any more.
        cp_async_wait_all();
        __syncwarp();
    #pragma unroll
        for (int bb = 0; bb < BW; ++bb) {
            float4 *part = reinterpret_cast<float4 *>(region) + bb * (TO / 4);
            const int E = -S[bb];
            const float f1 = pow2f(E / 2), f2 = pow2f(E - E / 2);
            const bool live = lane_ok && n > 0 && bb < nbw;
    #pragma unroll
            for (int c = 0; c < OPL / 4; ++c)
                part[NM ? part_chunk16(lane, c) : part_chunk(lane, c)] =
                    live ? make_float4((acc[bb][4 * c] * f1) * f2, (acc[bb][4 * c + 1] * f1) * f2,
                                       (acc[bb][4 * c + 2] * f1) * f2, (acc[bb][4 * c + 3] * f1) * f2)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncthreads();
        // Each thread owns chunks of 4 outputs of the tile (one, or two for the
        // 2:4 tile); for every batch row it sums the partial tiles of the warps of
        // that row's group and adds the sum into the workspace.
        if (NM) {
    #pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int q = tid + r * kThreads1; // chunk of the 2048-output tile
                const int l = q >> 4, c = q & 15;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    #pragma unroll
                for (int w = 0; w < kWarps1; ++w) {
                    const float4 u = reinterpret_cast<const float4 *>(
                        ring + (size_t)w * warp_region_bytes(BW, NM))[part_chunk16(l, c)];
                    v.x += u.x;
                    v.y += u.y;
                    v.z += u.z;
                    v.w += u.w;
                }
                if (n0 + 4 * q < p.N)
                    red_add_v4(p.ws_acc + n0 + 4 * q, v);
            }
        } else     if (BW == 1) {
            const int l = tid >> 3, c = tid & 7;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    #pragma unroll
            for (int w = 0; w < kWarps1; ++w) {
                const float4 u = reinterpret_cast<const float4 *>(
                    ring + (size_t)w * warp_region_bytes(BW))[part_chunk(l, c)];
                v.x += u.x;
                v.y += u.y;
                v.z += u.z;
                v.w += u.w;
            }
            if (n0 + 4 * tid < p.N)
                red_add_v4(p.ws_acc + n0 + 4 * tid, v);
        } else {
            const int l = tid >> 3, c = tid & 7;
            for (int b = 0; b < p.B; ++b) {
                const int w0 = (b / BW) * wpg, bb = b % BW;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int w = w0; w < w0 + wpg; ++w) {
                    const float4 u = reinterpret_cast<const float4 *>(
                        ring + (size_t)w * warp_region_bytes(BW))[bb * (kTileN1 / 4) + part_chunk(l, c)];
                    v.x += u.x;
                    v.y += u.y;
                    v.z += u.z;
                    v.w += u.w;
                }
                if (n0 + 4 * tid < p.N)
                    red_add_v4(p.ws_acc + (size_t)b * p.N + n0 + 4 * tid, v);
            }
        }

    }
}

// ---------------------------------------------------------------------------
// Host-side configuration
// ---------------------------------------------------------------------------

// The GEMV grid, then the split-K epilogue grid behind it.
template <typename Kern>
cudaError_t launch_gemv_and_finalize(Kern kern, int grid, int block, size_t smem,
                                     cudaStream_t stream, const KParams &kp)
{
    cudaError_t err = launch_pdl(kern, grid, block, smem, stream, kp);
    if (err != cudaSuccess || kp.p.accumulate)
        return err;
    return launch_finalize(kp.p, stream);
}

// Batch groups of warps for B > 1: ceil(B / 2) rounded up to 1, 2, 4 or 8.
int batch_groups(int B)
{
    const int need = (B + 1) / 2;
    int nb = 1;
    while (nb < need)
        nb *= 2;
    return nb;
}

template <int SRC, int BW, bool NM = false>
cudaError_t launch_gemv_t(KParams kp, int num_sms, cudaStream_t stream)
{
    const GemvProblem &p = kp.p;
    kp.nb = (BW == 1) ? 1 : batch_groups(p.B);
    const int bp = kp.nb * BW;
    kp.n_tiles = ceil_div(p.N, NM ? 2 * kTileN1 : kTileN1);
    kp.k_splits = std::max(1, num_sms / kp.n_tiles);
    const int G = p.K >> kp.lg;
    Smem1 L;
    for (;;) {
        kp.rows_cap = ceil_div(p.K, kp.k_splits) + 8;
        kp.span_cap = std::min(G, ceil_div(p.K, (long long)kp.k_splits << kp.lg) + 2);
        L = smem1_layout(kp.span_cap, kp.rows_cap, bp, BW, NM);
        // the threshold path handles at most 4 runs of 32 channels per warp
        // (the batch-1 threshold / GLU prologue keeps up to 4 runs of 32
        // channels per warp in registers; the batch-row union has no limit)
        const bool fused_select = (SRC == ROWS_THRESH || SRC == ROWS_GLU) && BW == 1;
        const bool runs_ok = !fused_select || (kp.rows_cap <= 4 * kThreads1);
        if ((L.total <= kMaxSmem && runs_ok) || kp.k_splits >= p.K / 8)
            break;
        kp.k_splits *= 2;
    }
    if (L.total > kMaxSmem ||
        ((SRC == ROWS_THRESH || SRC == ROWS_GLU) && BW == 1 && kp.rows_cap > 4 * kThreads1))
        return cudaErrorInvalidConfiguration;
    // Index list on a tile count that whole splits per tile cannot spread
    // over 90% of the SMs (e.g. 50 tiles: 100 of 148 CTAs), or that needs
    // more than one wave: one equal share of the (tile, list entry) space per
    // SM instead (segments, see gemv_kernel).
    if constexpr ((SRC == ROWS_LIST || (SRC == ROWS_THRESH && BW == 2)) && !NM) {
        const long long ctas = (long long)kp.n_tiles * kp.k_splits;
        if (kp.n_tiles <= num_sms && (10 * ctas < 9LL * num_sms || ctas > num_sms) &&
            (long long)kp.n_tiles * p.K < (1ll << 31)) {
            KParams ks = kp;
            // a share: at most this many list entries, or channels of one
            // tile's slice (threshold source)
            const int share = ceil_div((long long)kp.n_tiles * p.K, num_sms);
            ks.rows_cap = std::min(p.K, share) + 8;
            // scale/zero staged for the groups a share's rows touch (about
            // twice its rows at 50% sparsity, or its channels' groups), as
            // many as shared memory holds; the others are folded from global
            // memory
            ks.span_cap = std::min(G, ceil_div((SRC == ROWS_LIST ? 2LL : 1LL) * share,
                                               1LL << kp.lg) + 2);
            Smem1 LS = smem1_layout(ks.span_cap, ks.rows_cap, bp, BW, NM);
            while (ks.span_cap > 1 && LS.total > kMaxSmem) {
                --ks.span_cap;
                LS = smem1_layout(ks.span_cap, ks.rows_cap, bp, BW, NM);
            }
            if (LS.total <= kMaxSmem)
                return launch_gemv_and_finalize(gemv_kernel<SRC, BW, NM, true>, num_sms,
                                                kThreads1, LS.total, stream, ks);
        }
    }
    return launch_gemv_and_finalize(gemv_kernel<SRC, BW, NM>, kp.n_tiles * kp.k_splits,
                                    kThreads1, L.total, stream, kp);
}

template <int SRC>
cudaError_t launch_src(KParams kp, int num_sms, cudaStream_t stream)
{
    if (kp.p.keep) // the 2:4 layout (batch 1 only, checked by the API)
        return launch_gemv_t<SRC, 1, true>(kp, num_sms, stream);
    if (kp.p.B == 1)
        return launch_gemv_t<SRC, 1>(kp, num_sms, stream);
    return launch_gemv_t<SRC, 2>(kp, num_sms, stream);
}

} // namespace

cudaError_t launch_finalize(const GemvProblem &p, cudaStream_t stream)
{
    const int quads = std::max(p.B * (p.N / 4), p.zero_extra_n / 4);
    const int fgrid = std::max(1, std::min(ceil_div(quads, 256), 148));
    switch (p.epilogue) {
    case EPI_GLU_SILU: return launch_pdl(finalize_kernel<EPI_GLU_SILU>, fgrid, 256, 0, stream, p);
    case EPI_GLU_RELU: return launch_pdl(finalize_kernel<EPI_GLU_RELU>, fgrid, 256, 0, stream, p);
    default: return launch_pdl(finalize_kernel<EPI_PLAIN>, fgrid, 256, 0, stream, p);
    }
}

size_t gemv_workspace_bytes(int N, int B)
{
    const size_t acc = (size_t)B * N * sizeof(float);
    return (acc + 255) / 256 * 256;
}

cudaError_t launch_gemv(const GemvProblem &p, int num_sms, cudaStream_t stream)
{
    KParams kp{};
    kp.p = p;
    kp.lg = __builtin_ctz((unsigned)p.group);
    // B > 4 over the plain layout: the tensor-core kernel. Up to 4 rows the
    // CUDA-core kernel (two batch rows per warp, one FMA per code and row)
    // measured faster; from 5 its cost steps up (a third batch group of
    // warps) and keeps growing with the rows.
    if (p.B > 4 && !p.keep &&
        (p.source == ROWS_LIST || p.source == ROWS_DENSE || p.source == ROWS_MASK ||
         p.source == ROWS_THRESH))
        return launch_gemv_mma(p, num_sms, stream);
    switch (p.source) {
    case ROWS_LIST: return launch_src<ROWS_LIST>(kp, num_sms, stream);
    case ROWS_DENSE: return launch_src<ROWS_DENSE>(kp, num_sms, stream);
    case ROWS_MASK: return launch_src<ROWS_MASK>(kp, num_sms, stream);
    case ROWS_GLU: return launch_gemv_t<ROWS_GLU, 1>(kp, num_sms, stream); // batch 1
    default:
        // the API admits the 2:4 threshold path at B = 1 only
        if (p.keep)
            return launch_gemv_t<ROWS_THRESH, 1, true>(kp, num_sms, stream);
        if (p.B == 1)
            return launch_gemv_t<ROWS_THRESH, 1>(kp, num_sms, stream);
        return launch_gemv_t<ROWS_THRESH, 2>(kp, num_sms, stream);
    }
}

} // namespace sgq
