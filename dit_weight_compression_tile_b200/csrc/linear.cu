// The decode fused into a tcgen05 GEMM: ep_linear_fused ("EntroPack API reference",
// CompressedLinear and CompressedFP8Linear / CompressedINT8Linear reconstruct the weight for every
// forward call; here it goes from the stream into the tensor cores' operand slices in shared memory
// and never reaches global memory).  The stream is GEMM-ordered (every tile one 128 x 64 tile of W);
// the tile decode is the one of decode_core.cuh with a sink that writes operand slices.
#include <mutex>

#include "decode_core.cuh"

namespace ep {
namespace {

// ------------------------------------------------------------------ the decode fused into a GEMM
// Y^T = W X^T for a weight W (N x K) held as a GEMM-ordered stream (EP_LAYOUT_GEMM): each stream tile
// is one 128 x 64 tile of W, tiles in band-major order (a band: 128 output features, all K tiles).
// Each CTA (one per SM) takes a range of tiles (TileMap): a range of one band's K tiles, or, where
// whole bands would leave SMs idle, an even share of all tiles that may span two or more bands.
// Warps 0 .. S-1 decode, one tile at a time each: a bulk copy of the stream tile into the warp's
// buffer, the matching slice of X (tokens padded to a multiple of 16: BF16 activations, or their
// 8-bit codes) into the warp's X buffer, then the tile's 32 steps.  Every 8 steps (16 for 8-bit
// codes) complete a K-slice of the tile, 128 features x 32 bytes, which goes to one of the warp's
// two 4 KB slice buffers (a ring) and is announced on that buffer's `full` barrier.  Warp S issues
// the tensor-core work: for each round of tiles, slice by slice, warp by warp (a fixed order, so
// the sums are the same on every call), one tcgen05.mma (M = 128 features, N = tokens, K = 16 BF16
// or 32 codes, A = the W slice, B = the X slice, both K-major) into the tensor-memory accumulator
// of the tile's band (one per band the CTA touches), committed to the slice buffer's `empty`
// barrier.  After the last MMA, warps 0..3 read the accumulators out of tensor memory into
// the CTA's partial sums; the last CTA to finish a band adds the partial sums of the CTAs that
// touched it in CTA order (the same sums on every call), scales, adds the bias, rounds once to BF16
// and writes the band's part of Y.
constexpr uint32_t kLinMaxWarps = 15;       // decoding warps per CTA
constexpr uint32_t kLinSlice = 128u * 16u * 2u;  // one 128 x 16 BF16 K-slice of a W tile
constexpr uint32_t kLinBarBytes = 40;       // per decoding warp: full[2], empty[2], copy

// Which tiles each CTA takes (tiles in band-major order, KT per band): either band-aligned (each
// band's K tiles split into `splits` ranges of ktps, CTA c = band * splits + split) or spread evenly
// (CTA c takes [c T / C, (c + 1) T / C), which may span bands).  first(c): CTA c's first tile
// (first(C) = T); cta_of(t): the CTA holding tile t.
struct TileMap {
    uint32_t T, C, KT, splits, ktps, aligned;
    __host__ __device__ __forceinline__ uint32_t first(uint32_t c) const {
        if (aligned) return (c / splits) * KT + min((c % splits) * ktps, KT);
        return uint32_t(uint64_t(c) * T / C);
    }
    __host__ __device__ __forceinline__ uint32_t cta_of(uint32_t t) const {
        if (aligned) return (t / KT) * splits + (t % KT) / ktps;
        return uint32_t((uint64_t(t + 1) * C - 1) / T);  // the largest c with first(c) <= t
    }
};

struct LinParams {
    Params dp;                 // the stream (tiles, tables, row factors, status)
    const uint16_t *x;         // activations, BF16, M x cols row-major
    float *part;               // partial sums (fp32, int32 for INT8): C x nacc slots of M x 128
    uint32_t *count;           // per band: CTAs done (zero between calls)
    const uint16_t *bias;      // nullable, BF16, N
    uint16_t *y;               // BF16, M x N
    TileMap map;               // the CTAs' tile ranges (map.C CTAs: the grid)
    uint32_t nacc;             // partial-sum slots per CTA (most bands a CTA touches)
    const uint8_t *xq;         // code containers: the activations' 8-bit codes, M x cols
    const float *xscale;       // code containers: the activations' per-token scales
    const float *wscale;       // code containers: the weight's per-row scales (from the stream)
    uint32_t M, N;             // tokens, output features (rows of W)
    uint32_t npad;             // tokens padded to a multiple of 16 (the MMA's N)
    uint32_t idesc;            // the MMA's instruction descriptor
    uint32_t tmem_cols;        // tensor-memory columns of the accumulator (a power of 2, >= 32)
    uint32_t KT;               // K tiles per band (cols / 64)
    uint32_t S;                // decoding warps
    uint32_t tile_buf;         // bytes of a stream-tile buffer
    uint32_t off_bars, off_tile, off_w, off_x;  // shared-memory layout (offsets from the dynamic base)
};

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// UMMA shared-memory descriptor of a K-major operand without swizzle at shared address a: 8 x 16-byte
// core matrices, `lbo` bytes apart along K and `sbo` bytes apart along M / N (both in 16-byte
// units), descriptor version 1, layout type 0
__device__ __forceinline__ uint64_t umma_desc_plain(uint32_t a, uint32_t lbo, uint32_t sbo) {
    return uint64_t((a >> 4) & 0x3fffu) | (uint64_t((lbo >> 4) & 0x3fffu) << 16) |
           (uint64_t((sbo >> 4) & 0x3fffu) << 32) | (uint64_t(1) << 46);
}

// where a decoding warp's steps go.  A K-slice is 128 rows x 32 bytes of the tile (16 BF16 weights or
// 32 8-bit codes: the K extent of one MMA), stored as no-swizzle K-major core matrices: row r's
// 16-byte chunk c at (r / 8) 256 + 128 c + 16 (r mod 8).  Step k writes 8 weights of row
// 32 (k mod 4) + lane at column block k / 4, so BF16 tiles complete a slice every 8 steps (4 slices
// per tile), 8-bit tiles every 16 (2 slices); slice j of the warp's round-th tile is its use
// U round + j (U slices per tile) and lives in ring buffer j mod 2.
template <int DT>
struct SliceSink {
    static constexpr uint32_t kSteps = DT == EP_BF16 ? 8u : 16u;  // steps per slice
    static constexpr uint32_t kUses = 32u / kSteps;                // slices per tile
    uint32_t ring;   // shared address of the warp's two slice buffers
    uint32_t full;   // full[0]; full[1] = full + 8, empty[j] = full + 16 + 8 j
    uint32_t round;  // the warp's tile number
    __device__ __forceinline__ bool begin(uint32_t k) const {
        // BF16 slices 2 and 3 reuse the buffers of slices 0 and 1: wait for their MMAs (use u - 2);
        // the buffers of a tile's first two slices were freed before the tile started
        if (k % kSteps != 0 || k < 2u * kSteps) return true;
        const uint32_t u = kUses * round + k / kSteps;
        return mbar_wait(full + 16u + 8u * (u & 1u), ((u - 2u) >> 1) & 1u);
    }
    __device__ __forceinline__ void put(uint32_t k, uint32_t lane, Packer<DT> &pk) const {
        const uint32_t r = 32u * (k & 3u) + lane, slot = (k / kSteps) & 1u;
        uint32_t off;
        if constexpr (DT == EP_BF16)
            off = ((k >> 2) & 1u) * 128u;  // 16 bytes per step: chunk (k / 4) mod 2
        else
            off = ((k >> 3) & 1u) * 128u + ((k >> 2) & 1u) * 8u;  // 8 bytes per step
        pk.store_shared(ring + slot * kLinSlice + (r >> 3) * 256u + (r & 7u) * 16u + off);
    }
    __device__ __forceinline__ void end(uint32_t k, uint32_t lane) const {
        if (k % kSteps != kSteps - 1u) return;
        // the slice, written through the generic proxy, becomes visible to the tensor cores
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(full + 8u * ((k / kSteps) & 1u));
    }
};

// the X operand: BF16 (K = 16 per MMA) or the 8-bit codes of the quantized activations (K = 32);
// either way 32 bytes of a row per MMA, row n's 16-byte chunk c of a K tile at
// (n / 8) 8 XB + 128 c + 16 (n mod 8), XB the row's bytes per K tile
template <int DT>
struct XOperand {
    static constexpr uint32_t kRowBytes = DT == EP_BF16 ? 128u : 64u;  // one K tile (64 inputs) of a row
};

template <int DT, int MODE>
__global__ void __launch_bounds__((kLinMaxWarps + 1) * 32, 1) linear_kernel(const __grid_constant__ LinParams P) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr uint32_t XB = XOperand<DT>::kRowBytes;
    const Params &p = P.dp;
    constexpr uint32_t kTables = uint32_t(MODE == kPaired ? kPairedTableBytes : kLutBytes);
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5, S = P.S;
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const uint32_t lut = base;
    auto wbar = [&](uint32_t w) { return base + P.off_bars + kLinBarBytes * w; };  // full[2], empty[2], copy
    const uint32_t tbar = base + P.off_bars + kLinBarBytes * S, done = tbar + 8u, tmem_slot = tbar + 16u;
    auto ring = [&](uint32_t w) { return base + P.off_w + 2u * kLinSlice * w; };
    auto xbuf = [&](uint32_t w) { return base + P.off_x + P.npad * XB * w; };
    auto tbuf = [&](uint32_t w) { return base + P.off_tile + P.tile_buf * w; };
    const uint32_t cta = blockIdx.x;
    const uint32_t t0 = P.map.first(cta);
    const uint32_t nkt = P.map.first(cta + 1) - t0;  // >= 1: the plan leaves no CTA without tiles
    const uint32_t b0 = t0 / P.KT, nband = (t0 + nkt - 1) / P.KT - b0 + 1;  // bands touched, <= P.nacc

    if (threadIdx.x == 0) {
        for (uint32_t w = 0; w < S; ++w)
            for (uint32_t i = 0; i < 5; ++i) mbar_init(wbar(w) + 8u * i, 1);
        mbar_init(tbar, 1);
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async();
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == S) {  // the accumulator's tensor memory (the whole warp allocates)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot),
                     "r"(P.tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (threadIdx.x == 0) {
        mbar_expect(tbar, kTables);
        bulk_g2s(lut, p.tables, kTables, tbar);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = lds32(tmem_slot);
    bool ok = mbar_wait(tbar, 0);
    uint32_t err = ok ? 0u : uint32_t(EP_DEC_TIMEOUT);

    if (warp < S) {
        // ---- decoding warps: tiles t0 + j, j = warp, warp + S, ... of the CTA's range
        SliceSink<DT> sink{ring(warp), wbar(warp), 0u};
        const uint32_t copyb = wbar(warp) + 32u;
        for (uint32_t j = warp; j < nkt && ok; j += S, ++sink.round) {
            const uint32_t t = t0 + j, kt = t % P.KT;
            // the MMAs of the previous tile (its last slice, use U round - 1, in ring buffer 1, and
            // so all before it) are done: the X buffer and both slice buffers are free
            if (sink.round > 0 && !mbar_wait(wbar(warp) + 24u, ((SliceSink<DT>::kUses * sink.round - 1u) >> 1) & 1u)) {
                err |= EP_DEC_TIMEOUT;
                break;
            }
            const uint32_t beg = __ldg(p.dir + t), end = __ldg(p.dir + t + 1), bytes = (end - beg) * 16u;
            if (end < beg + uint32_t(kTileHead / 16) || uint64_t(end) > p.tile_units || bytes + kSlack > P.tile_buf) {
                err |= EP_DEC_BAD_TILE;
                break;
            }
            if (lane == 0) {
                fence_proxy_async();
                mbar_expect(copyb, bytes);
                bulk_g2s(tbuf(warp), p.tiles + size_t(beg) * 16, bytes, copyb);
            }
            // X rows n < npad, inputs 64 kt .. + 63 (zero for n >= M): XB / 16 lanes per row, 16 bytes
            // each (BF16 activations, or their 8-bit codes quantized by the launch before this one)
            constexpr uint32_t kLanesPerRow = XB / 16u;
            const uint32_t xb = xbuf(warp), c = lane % kLanesPerRow;
            const uint8_t *xrow = DT == EP_BF16 ? reinterpret_cast<const uint8_t *>(P.x) + 128u * kt : P.xq + 64u * kt;
            const size_t xstride = DT == EP_BF16 ? 2u * p.cols : p.cols;
            for (uint32_t n = lane / kLanesPerRow; n < P.npad; n += 32u / kLanesPerRow) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (n < P.M) v = __ldg(reinterpret_cast<const uint4 *>(xrow + size_t(n) * xstride) + c);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xb + (n >> 3) * 8u * XB + c * 128u +
                                                                              (n & 7u) * 16u),
                             "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                             : "memory");
            }
            if (!mbar_wait(copyb, sink.round & 1u)) {
                err |= EP_DEC_TIMEOUT;
                break;
            }
            const uint32_t e = decode_tile<DT, kRowsGemm, MODE, true, uint32_t, SliceSink<DT>>(
                p, lut, tbuf(warp), bytes, t, lane, &sink);
            err |= e;
            if (__any_sync(0xffffffffu, e != 0)) break;  // the tile's slices may be missing: stop here
        }
    } else if (warp == S) {
        // ---- the MMA issuer: round by round, slice by slice, warp by warp
        constexpr uint32_t U = SliceSink<DT>::kUses;
        const uint32_t rounds = (nkt + S - 1) / S;
        uint32_t started = 0;  // the accumulators (bands) that have had their first MMA
        for (uint32_t r = 0; r < rounds && ok; ++r) {
            // the band (accumulator) of the round's first tile, and the tile's place in it
            const uint32_t ar = (t0 + r * S) / P.KT - b0, kr = (t0 + r * S) % P.KT;
            for (uint32_t sl = 0; sl < U && ok; ++sl) {
                uint32_t a = ar, kin = kr;
                for (uint32_t w = 0; w < S && r * S + w < nkt; ++w, ++kin) {
                    if (kin == P.KT) {  // this warp's tile starts the next band
                        kin = 0;
                        ++a;
                    }
                    const uint32_t u = U * r + sl, fb = wbar(w) + 8u * (u & 1u);
                    if (!mbar_wait(fb, (u >> 1) & 1u)) {
                        err |= EP_DEC_TIMEOUT;
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t d = tmem + a * P.npad;  // the accumulator of the tile's band
                    if (lane == 0) {
                        const uint64_t da = umma_desc_plain(ring(w) + (u & 1u) * kLinSlice, 128u, 256u);
                        const uint64_t db = umma_desc_plain(xbuf(w) + 256u * sl, 128u, 8u * XB);
                        const uint32_t acc = (started >> a) & 1u;
                        if constexpr (DT == EP_BF16)
                            asm volatile(
                                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                                "l"(da), "l"(db), "r"(P.idesc), "r"(acc)
                                : "memory");
                        else if constexpr (DT == EP_INT8)
                            asm volatile(
                                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                                "l"(da), "l"(db), "r"(P.idesc), "r"(acc)
                                : "memory");
                        else
                            asm volatile(
                                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                                "l"(da), "l"(db), "r"(P.idesc), "r"(acc)
                                : "memory");
                        asm volatile(
                            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                fb + 16u)
                            : "memory");
                    }
                    started |= 1u << a;
                    __syncwarp();
                }
            }
        }
        if (lane == 0)
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(done)
                         : "memory");
        __syncwarp();
    }
    // ---- epilogue: warp q < 4 reads tensor-memory lanes 32 q .. 32 q + 31 (features) of each band's
    // accumulator, one column per token, into the CTA's partial-sum slot of that band: M rows of the
    // band's 128 features (each warp writes 128 contiguous bytes per token)
    if (warp < 4) {
        if (!mbar_wait(done, 0)) err |= EP_DEC_TIMEOUT;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        for (uint32_t a = 0; a < nband; ++a) {
            uint32_t *dst = reinterpret_cast<uint32_t *>(P.part) + size_t(cta * P.nacc + a) * P.M * 128u + 32u * warp +
                            lane;
            for (uint32_t c0 = 0; c0 < P.npad; c0 += 16u) {
                uint32_t r[16];
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                    "%13, %14, %15}, [%16];"
                    : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                      "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                      "=r"(r[15])
                    : "r"(tmem + ((32u * warp) << 16) + a * P.npad + c0));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                for (uint32_t i = 0; i < 16u; ++i)  // fp32 sums, or the int32 sums of the INT8 MMA, as bits
                    if (c0 + i < P.M) dst[size_t(c0 + i) * 128u] = r[i];
            }
        }
    }
    if (err && p.status && lane == 0) atomicOr(p.status, err);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // the partial sums are visible device-wide before this CTA counts itself done
    __threadfence();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == S) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(P.tmem_cols)
                     : "memory");
    }
    // ---- count this CTA in each band it touched; the band's last CTA (the one that completes its
    // count: every CTA from the one holding the band's first tile to the one holding its last) adds
    // the band's partial sums
    if (threadIdx.x == 0) {
        uint32_t last = 0;
        for (uint32_t a = 0; a < nband; ++a) {
            const uint32_t b = b0 + a;
            const uint32_t lo = P.map.cta_of(b * P.KT), hi = P.map.cta_of((b + 1) * P.KT - 1u);
            if (atomicAdd(P.count + b, 1u) == hi - lo) last |= 1u << a;
        }
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(tmem_slot), "r"(last) : "memory");
    }
    __syncthreads();
    const uint32_t last = lds32(tmem_slot);
    if (last == 0u) return;
    __threadfence();
    // four features per thread and step; the loads of up to eight CTAs' partials are issued before
    // their additions, which stay in CTA order (INT8: exact int32 sums).  BF16: y = RNE(sum + bias).
    // Codes: y = RNE(fp32(fp32(sum) s_x) s_w), then with a bias RNE(y + bias): the order of the
    // per-row-quantized layers' own arithmetic
    using Acc = typename std::conditional<DT == EP_INT8, int32_t, float>::type;
    using Acc4 = typename std::conditional<DT == EP_INT8, int4, float4>::type;
    for (uint32_t a = 0; a < nband; ++a) {
        if (!((last >> a) & 1u)) continue;
        const uint32_t b = b0 + a;
        const uint32_t lo = P.map.cta_of(b * P.KT), hi = P.map.cta_of((b + 1) * P.KT - 1u);
        // CTA lo may start in an earlier band (its slot for b is further on); every later contributor
        // starts inside band b, so band b is its first slot
        const uint32_t slot_lo = lo * P.nacc + (b - P.map.first(lo) / P.KT);
        for (uint32_t i = threadIdx.x; i < P.M * 32u; i += blockDim.x) {
            const uint32_t m = i >> 5, f = 4u * (i & 31u), n = 128u * b + f;
            Acc acc[4] = {Acc(0), Acc(0), Acc(0), Acc(0)};
            for (uint32_t c0 = lo; c0 <= hi; c0 += 8u) {
                Acc4 v[8];
#pragma unroll
                for (uint32_t j = 0; j < 8u; ++j)
                    if (c0 + j <= hi) {
                        const uint32_t c = c0 + j;
                        const uint32_t slot = c == lo ? slot_lo : c * P.nacc;
                        v[j] = __ldcg(reinterpret_cast<const Acc4 *>(P.part + (size_t(slot) * P.M + m) * 128u + f));
                    }
#pragma unroll
                for (uint32_t j = 0; j < 8u; ++j)
                    if (c0 + j <= hi) {
                        acc[0] += v[j].x;
                        acc[1] += v[j].y;
                        acc[2] += v[j].z;
                        acc[3] += v[j].w;
                    }
            }
            uint16_t *dst = P.y + size_t(m) * P.N + n;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float yv;
                if constexpr (DT == EP_BF16) {
                    yv = acc[j];
                    if (P.bias) yv += __uint_as_float(uint32_t(P.bias[n + j]) << 16);
                } else {
                    const float fa = DT == EP_INT8 ? __int2float_rn(int32_t(acc[j])) : float(acc[j]);
                    yv = __fmul_rn(__fmul_rn(fa, P.xscale[m]), __ldg(P.wscale + n + j));
                    if (P.bias)
                        yv = __bfloat162float(__float2bfloat16_rn(yv)) + __uint_as_float(uint32_t(P.bias[n + j]) << 16);
                }
                const __nv_bfloat16 h = __float2bfloat16_rn(yv);
                dst[j] = *reinterpret_cast<const uint16_t *>(&h);
            }
        }
        if (threadIdx.x == 0) P.count[b] = 0u;  // ready for the next call
    }
}

// The activations of a per-row-quantized layer: per token, scale = amax / 127 (INT8) or / 448 (FP8
// E4M3), 1 for an all-zero row; codes = x / scale rounded to nearest even and clamped to [-127, 127]
// (INT8), or clamped to [-448, 448] and rounded to E4M3 (FP8).  One CTA per token.
template <int DT>
__global__ void __launch_bounds__(256) quantize_x_kernel(const uint16_t *x, uint32_t K, uint8_t *xq, float *xscale) {
    __shared__ float part[8];
    const uint32_t m = blockIdx.x;
    const uint16_t *row = x + size_t(m) * K;
    float amax = 0.0f;
    for (uint32_t k = threadIdx.x; k < K; k += blockDim.x) amax = fmaxf(amax, fabsf(__uint_as_float(uint32_t(row[k]) << 16)));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
    if ((threadIdx.x & 31u) == 0) part[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = part[0];
    for (uint32_t w = 1; w < (blockDim.x >> 5); ++w) amax = fmaxf(amax, part[w]);
    const float scale = amax > 0.0f ? __fdiv_rn(amax, DT == EP_INT8 ? 127.0f : 448.0f) : 1.0f;
    if (threadIdx.x == 0) xscale[m] = scale;
    uint8_t *out = xq + size_t(m) * K;
    for (uint32_t k = threadIdx.x; k < K; k += blockDim.x) {
        const float v = __fdiv_rn(__uint_as_float(uint32_t(row[k]) << 16), scale);
        if constexpr (DT == EP_INT8)
            out[k] = uint8_t(int8_t(__float2int_rn(fminf(fmaxf(rintf(v), -127.0f), 127.0f))));
        else
            out[k] = uint8_t(__nv_cvt_float_to_fp8(fminf(fmaxf(v, -448.0f), 448.0f), __NV_SATFINITE, __NV_E4M3));
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- the fused GEMM's launch plan.  The T = bands x KT tiles go to CTAs (one per SM) either
// band-aligned (each band's K tiles split so that about one wave of CTAs runs) or spread evenly over
// one wave (more CTAs when one would touch more bands than tensor memory holds accumulators for);
// the plan takes the even spread only when it needs fewer rounds of tiles per decoding warp (times
// waves), since aligned CTAs have one accumulator and fewer contributors per band.  Shared memory =
// tables, barriers, then per decoding warp a stream-tile buffer, two W slice buffers and an X
// buffer; decoding warps: as many as fit, then as few as give the same number of rounds.
struct LinPlan {
    TileMap map;
    uint32_t nbands, KT, L, nacc, S, npad, tmem_cols, tile_buf, off_bars, off_tile, off_w, off_x;
    uint32_t xrow;  // bytes of one token's K tile in the X buffer: 128 (BF16) or 64 (8-bit codes)
    bool codes;     // an INT8 / FP8 container: the activations are quantized per token first
    size_t smem;
};

LinPlan lin_plan(const ep_info *info, int sms, int64_t m) {
    LinPlan P{};
    P.nbands = uint32_t(info->rows / 128);
    P.KT = uint32_t(info->cols / 64);
    const uint32_t T = P.nbands * P.KT;
    P.npad = uint32_t((m + 15) / 16 * 16);
    P.codes = info->container_dtype != EP_BF16;
    P.xrow = P.codes ? 64u : 128u;
    P.tile_buf = uint32_t((info->max_tile_nbytes + kSlack + 15) & ~uint64_t(15));
    const uint32_t tables = uint32_t(info->paired ? kPairedTableBytes : kLutBytes);
    auto layout = [&](uint32_t S) {
        P.S = S;
        P.off_bars = tables;
        P.off_tile = (P.off_bars + kLinBarBytes * S + 24u + 15u) & ~15u;
        P.off_w = (P.off_tile + S * P.tile_buf + 127u) & ~127u;
        P.off_x = P.off_w + S * 2u * kLinSlice;
        P.smem = size_t(P.off_x) + size_t(S) * P.npad * P.xrow;
    };
    uint32_t smax = kLinMaxWarps;  // decoding warps that fit beside the tables
    for (layout(smax); smax > 1 && P.smem > kSmemLimit; layout(--smax)) {
    }
    auto warps_for = [&](uint32_t L) {  // as few warps as give the fewest rounds
        const uint32_t S = std::min(smax, L), rounds = (L + S - 1) / S;
        return (L + rounds - 1) / rounds;
    };
    auto most_bands = [&](const TileMap &M) {
        uint32_t n = 0;
        for (uint32_t c = 0; c < M.C; ++c) n = std::max(n, (M.first(c + 1) - 1) / P.KT - M.first(c) / P.KT + 1);
        return n;
    };
    const uint32_t waves_sm = uint32_t(std::max(sms, 1));
    // band-aligned
    TileMap A{T, 0, P.KT, 0, 0, 1};
    uint32_t splits_max = P.nbands < waves_sm ? waves_sm / P.nbands : 1u;
    splits_max = std::max(1u, std::min(splits_max, P.KT));
    A.ktps = (P.KT + splits_max - 1) / splits_max;
    A.splits = (P.KT + A.ktps - 1) / A.ktps;
    A.C = P.nbands * A.splits;
    const uint32_t SA = warps_for(A.ktps);
    const uint32_t cost_a = ((A.ktps + SA - 1) / SA) * ((A.C + waves_sm - 1) / waves_sm);
    // spread evenly
    TileMap E{T, std::min(waves_sm, T), P.KT, 1, P.KT, 0};
    uint32_t nacc_e = most_bands(E);
    while (nacc_e * P.npad > 512u && E.C < T) {
        E.C = std::min(T, 2u * E.C);
        nacc_e = most_bands(E);
    }
    const uint32_t LE = (T + E.C - 1) / E.C;
    const uint32_t SE = warps_for(LE);
    const uint32_t cost_e = ((LE + SE - 1) / SE) * ((E.C + waves_sm - 1) / waves_sm);
    if (cost_e < cost_a) {
        P.map = E;
        P.L = LE;
        P.nacc = nacc_e;
        layout(SE);
    } else {
        P.map = A;
        P.L = A.ktps;
        P.nacc = 1;
        layout(SA);
    }
    P.tmem_cols = 32;
    while (P.tmem_cols < P.nacc * P.npad) P.tmem_cols *= 2;
    // more than half an SM's shared memory: one CTA per SM, so no CTA waits for another's tensor memory
    P.smem = std::max(P.smem, kSmemLimit / 2 + 1024);
    return P;
}
// the plan fits the shared memory (the accumulators fit the 512 columns of tensor memory by the
// choice of C)
bool lin_fits(const LinPlan &P) { return P.smem <= kSmemLimit && P.tmem_cols <= 512u; }

// the caller's scratch: the partial sums (CTAs x nacc slots of m x 128, fp32 or int32), one counter per
// band, and for code containers the activations' codes (m x K bytes) and per-token scales (m floats)
size_t lin_count_offset(const LinPlan &P, int64_t m) {
    return (size_t(P.map.C) * P.nacc * size_t(m) * 128u * sizeof(float) + 15u) & ~size_t(15);
}
size_t lin_xq_offset(const LinPlan &P, int64_t m) {
    return (lin_count_offset(P, m) + size_t(P.nbands) * 4u + 15u) & ~size_t(15);
}
size_t lin_xscale_offset(const LinPlan &P, int64_t m) {
    return (lin_xq_offset(P, m) + size_t(m) * P.KT * 64u + 15u) & ~size_t(15);
}
size_t lin_work_bytes(const LinPlan &P, int64_t m) {
    return P.codes ? lin_xscale_offset(P, m) + size_t(m) * 4u : lin_count_offset(P, m) + size_t(P.nbands) * 4u;
}

}  // namespace
}  // namespace ep

// ------------------------------------------------------------------ ep_linear_fused
namespace ep {
namespace {

struct SmCache {
    std::mutex mu;
    int sms[64] = {0};
};
SmCache g_sms;

int device_sms(int *device, int *sms) {
    if (cudaGetDevice(device) != cudaSuccess || *device < 0 || *device >= 64) return EP_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_sms.mu);
    if (!g_sms.sms[*device] &&
        cudaDeviceGetAttribute(&g_sms.sms[*device], cudaDevAttrMultiProcessorCount, *device) != cudaSuccess)
        return EP_ERR_CUDA;
    *sms = g_sms.sms[*device];
    return EP_OK;
}

bool linear_ok(const ep_info *info, int64_t m) {
    return info && info->layout == 1 &&
           (info->container_dtype == EP_BF16 || info->container_dtype == EP_INT8 ||
            info->container_dtype == EP_FP8_E4M3) &&
           m >= 1 && m <= 128 && check_info(info) == EP_OK;
}

struct LinCache {
    std::mutex mu;
    size_t smem_set[64][9] = {};  // [device][3 container + coding mode]
};
LinCache g_lin;

}  // namespace
}  // namespace ep

extern "C" int ep_linear_fused_plan(const ep_info *info, int64_t m, int32_t sms, ep_linear_plan *out) {
    using namespace ep;
    if (!out || sms < 1 || !linear_ok(info, m)) return EP_ERR_INVALID_ARG;
    const LinPlan L = lin_plan(info, sms, m);
    out->bands = L.nbands;
    out->ctas = L.map.C;
    out->tiles_per_cta = L.L;
    out->accumulators = L.nacc;
    out->spread = L.map.aligned ? 0u : 1u;
    out->splits = L.map.aligned ? L.map.splits : 0u;
    out->decoding_warps = L.S;
    out->threads = std::max(L.S + 1, 4u) * 32u;
    out->tokens_padded = L.npad;
    out->tmem_columns = L.tmem_cols;
    out->tile_buffer_bytes = L.tile_buf;
    out->smem_tables_bytes = L.off_bars;
    out->smem_barriers_offset = L.off_bars;
    out->smem_tiles_offset = L.off_tile;
    out->smem_slices_offset = L.off_w;
    out->smem_x_offset = L.off_x;
    out->smem_x_bytes_per_warp = L.npad * L.xrow;
    out->smem_bytes = L.smem;
    out->work_bytes = lin_work_bytes(L, m);
    return lin_fits(L) ? EP_OK : EP_ERR_UNSUPPORTED;
}

extern "C" size_t ep_linear_fused_workspace(const ep_info *info, int64_t m) {
    using namespace ep;
    if (!linear_ok(info, m)) return 0;
    int device, sms;
    if (device_sms(&device, &sms) != EP_OK) return 0;
    const LinPlan L = lin_plan(info, sms, m);
    return lin_work_bytes(L, m);
}

extern "C" int ep_linear_fused(const ep_info *info, const void *d_blob, const void *d_tables, const void *d_x,
                               int64_t m, const void *d_bias, void *d_y, void *d_work, size_t work_nbytes,
                               uint32_t *d_status, ep_stream_t stream) {
    using namespace ep;
    if (!d_blob || !d_tables || !d_x || !d_y || !d_work || !linear_ok(info, m)) return EP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_blob) | reinterpret_cast<uintptr_t>(d_tables) |
         reinterpret_cast<uintptr_t>(d_x) | reinterpret_cast<uintptr_t>(d_work)) & 15u)
        return EP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_y) & 1u || reinterpret_cast<uintptr_t>(d_bias) & 1u) return EP_ERR_INVALID_ARG;
    int device, sms;
    if (device_sms(&device, &sms) != EP_OK) return EP_ERR_CUDA;
    const LinPlan L = lin_plan(info, sms, m);
    if (work_nbytes < lin_work_bytes(L, m)) return EP_ERR_INVALID_ARG;
    // tiles too large for one warp's buffers beside the tables, or too many bands per CTA for the
    // accumulators of a large token count
    if (!lin_fits(L)) return EP_ERR_UNSUPPORTED;
    LinParams P;
    P.dp = params_of(info, d_blob, d_tables, nullptr, d_status);
    P.x = static_cast<const uint16_t *>(d_x);
    P.part = static_cast<float *>(d_work);
    P.count = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(d_work) + lin_count_offset(L, m));
    P.bias = static_cast<const uint16_t *>(d_bias);
    P.y = static_cast<uint16_t *>(d_y);
    P.map = L.map;
    P.nacc = L.nacc;
    P.M = uint32_t(m);
    P.N = uint32_t(info->rows);
    P.npad = L.npad;
    // the MMA's instruction descriptor: accumulator type (bits 4..5: 1 fp32, 2 int32), A and B types
    // (bits 7..9, 10..12: BF16 = 1 for kind::f16, signed = 1 for kind::i8, E4M3 = 0 for
    // kind::f8f6f4), both K-major, N = npad (bits 17..22: N / 8), M = 128 (bits 24..28: M / 16)
    const int dt = info->container_dtype;
    const uint32_t types = dt == EP_BF16 ? (1u << 4) | (1u << 7) | (1u << 10)
                           : dt == EP_INT8 ? (2u << 4) | (1u << 7) | (1u << 10)
                                           : (1u << 4);
    P.idesc = types | ((L.npad >> 3) << 17) | ((128u >> 4) << 24);
    P.tmem_cols = L.tmem_cols;
    P.KT = L.KT;
    P.S = L.S;
    P.tile_buf = L.tile_buf;
    P.off_bars = L.off_bars;
    P.off_tile = L.off_tile;
    P.off_w = L.off_w;
    P.off_x = L.off_x;
    uint8_t *work = static_cast<uint8_t *>(d_work);
    P.xq = L.codes ? work + lin_xq_offset(L, m) : nullptr;
    P.xscale = L.codes ? reinterpret_cast<const float *>(work + lin_xscale_offset(L, m)) : nullptr;
    P.wscale = L.codes ? reinterpret_cast<const float *>(static_cast<const uint8_t *>(d_blob) + info->off_scales)
                       : nullptr;
    const int mode = info->paired ? kPaired : (wide_fields(info) ? kWide : kNarrow);
    using Kern = void (*)(LinParams);
    // [container: BF16, INT8, FP8][coding mode]
    static const Kern kerns[3][3] = {
        {linear_kernel<EP_BF16, kNarrow>, linear_kernel<EP_BF16, kWide>, linear_kernel<EP_BF16, kPaired>},
        {linear_kernel<EP_INT8, kNarrow>, linear_kernel<EP_INT8, kWide>, linear_kernel<EP_INT8, kPaired>},
        {linear_kernel<EP_FP8_E4M3, kNarrow>, linear_kernel<EP_FP8_E4M3, kWide>, linear_kernel<EP_FP8_E4M3, kPaired>}};
    const int ci = dt == EP_BF16 ? 0 : (dt == EP_INT8 ? 1 : 2);
    const Kern kern = kerns[ci][mode];
    {
        std::lock_guard<std::mutex> g(g_lin.mu);
        size_t &set = g_lin.smem_set[device][3 * ci + mode];
        if (set < L.smem) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(L.smem)) != cudaSuccess)
                return EP_ERR_CUDA;
            set = L.smem;
        }
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (L.codes) {  // the activations' codes and scales, into the scratch
        float *xs = reinterpret_cast<float *>(work + lin_xscale_offset(L, m));
        uint8_t *xq = work + lin_xq_offset(L, m);
        const uint16_t *x = static_cast<const uint16_t *>(d_x);
        if (dt == EP_INT8)
            quantize_x_kernel<EP_INT8><<<unsigned(m), 256, 0, s>>>(x, uint32_t(info->cols), xq, xs);
        else
            quantize_x_kernel<EP_FP8_E4M3><<<unsigned(m), 256, 0, s>>>(x, uint32_t(info->cols), xq, xs);
        if (cudaGetLastError() != cudaSuccess) return EP_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(L.map.C);
    cfg.blockDim = dim3(std::max(L.S + 1, 4u) * 32);  // the epilogue needs warps 0..3
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, P) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
