// verify_greedy_ee.cu -- the greedy lossless verify with early exit: target
// rows after a sequence's first mismatch are not read.
//
// Sources: "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "Les chiffres qui comptent sur Qwen3.8-27B": greedy
// verification reproduces the target exactly; "DFlash 2: un drafter de 3.43×
// que cae a 1.45× bajo carga" (latenode.com), section "El desacuerdo empieza
// en las propias tablas del proveedor": acceptance length = tokens completed
// per verify step.  The result is the one of dflash2_verify_greedy:
//   t_j = argmax_v target[j][v] (lowest v on ties), n = first j with
//   draft_tok[j] != t_j (else G); out = draft_tok[0..n-1], t_n, -1 ...
// Only rows 0..n are needed, and row j mismatches exactly when some element
// of it has a larger (value, -index) key than the drafted token's.
//
// Work units are (row j, sequence b, 8 KB chunk) in that order and warp w of
// the grid takes units w, w + W, w + 2 W, ... (W warps), so every warp moves
// through the rows in step with the others: all sequences' row 0, then row 1,
// and so on.  A chunk whose (maximum, lowest index) key beats the drafted
// token's key marks its row as mismatched (one atomic maximum on the
// sequence's skip word, which encodes the lowest such row); a unit of a later
// row of that sequence is skipped when it would be brought in (no copy, no
// arithmetic) and only counted.  A row at or before the first mismatch is
// never skipped (nothing before it mismatches), so rows 0..n are complete
// when the sequence's last unit is counted, and the warp counting it decides
// the sequence from them.  Each warp streams through its own two ring slots
// (TMA bulk copies, ring.cuh); every wait is bounded.
#include <type_traits>

#include "common.cuh"
#include "greedy.cuh"
#include "ring.cuh"
#include "workspace.cuh"

namespace dfl {

constexpr int EE_MAX_TOK = 1024;  // drafted tokens (B G) the shared key table holds
constexpr int EE_MAX_SEQ = 1024;  // sequences the shared skip words hold

template <bool BF16>
__global__ void __launch_bounds__(RING_THREADS, 1) verify_greedy_ee_kernel(
    const void* __restrict__ target, int B, int G, int64_t V, int S, int64_t units,
    const int32_t* __restrict__ draft_tok, int32_t* __restrict__ n_accept,
    int32_t* __restrict__ out_tok, uint64_t* __restrict__ part, unsigned* __restrict__ counters,
    unsigned* __restrict__ skipw) {
    using Ch = ChunkT<BF16>;
    constexpr int ES = Ch::ES;
    constexpr int LEN = Ch::LEN;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t bars[2 * NCW];
    __shared__ uint64_t s_dkey[EE_MAX_TOK];  // the drafted tokens' keys [B][G]
    __shared__ unsigned s_skip[EE_MAX_SEQ];  // this CTA's view of the skip words [B]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // every drafted token's key in shared memory (one round of loads per CTA),
    // so no unit waits on a dependent global load before its copy is issued
    for (int i = threadIdx.x; i < B * G; i += blockDim.x) {
        const int64_t b = i / G, j = i - b * G;
        const int32_t d = draft_tok[i];
        uint64_t dk = 0ull;  // a token outside [0, V): every chunk beats it (a mismatch)
        if ((uint32_t)d < (uint64_t)V) {
            const int64_t o = (b * (G + 1) + j) * V + d;
            const float x = BF16 ? __uint_as_float((uint32_t)((const uint16_t*)target)[o] << 16)
                                 : ((const float*)target)[o];
            dk = make_key(x, (uint32_t)d);
        }
        s_dkey[i] = dk;
    }
    for (int i = threadIdx.x; i < B; i += blockDim.x) s_skip[i] = 0u;
    __syncthreads();
    const int64_t gw = (int64_t)blockIdx.x * NCW + warp, nw = (int64_t)gridDim.x * NCW;
    const int n = gw < units ? (int)((units - 1 - gw) / nw + 1) : 0;
    const int64_t per_row = (int64_t)B * S;
    WarpRing r{ring + 2 * warp * SLOT_BYTES, smem_u32(&bars[2 * warp])};
    if (lane == 0) {
        mbar_init(r.bar, 1);
        mbar_init(r.bar + 8, 1);
        mbar_fence_init();
    }
    __syncwarp();
    // per ring slot: the unit it holds, whether it was skipped, the drafted
    // token's key of its row and the parity its copy completes
    int64_t sb[2] = {0, 0};
    int sj[2] = {0, 0}, sc[2] = {0, 0};
    bool skip[2] = {true, true};
    uint64_t dkey[2] = {0ull, 0ull};
    uint32_t issued[2] = {0u, 0u};
    auto unit_of = [&](int k, int64_t& b, int& j, int& c) {
        const int64_t u = gw + (int64_t)k * nw;
        j = (int)(u / per_row);
        const int64_t rem = u - (int64_t)j * per_row;
        b = rem / S;
        c = (int)(rem - b * S);
    };
    // bring unit k into slot S_ (= k & 1, a compile-time constant so the
    // per-slot state stays in registers); seen: a value of the sequence's
    // global skip word read earlier (or 0)
    auto bring = [&](auto S_, int k, unsigned seen) {
        constexpr int s = decltype(S_)::value;
        int64_t b;
        int j, c;
        unit_of(k, b, j, c);
        sb[s] = b;
        sj[s] = j;
        sc[s] = c;
        // any lower bound of the skip word is safe: skipping less is never wrong
        const unsigned w = max(seen, *(volatile unsigned*)&s_skip[b]);
        skip[s] = j + w > (unsigned)(G + 1);
        dkey[s] = (j < G) ? s_dkey[b * G + j] : ~0ull;  // row G has no drafted token
        if (!skip[s]) {
            const int64_t v0 = (int64_t)c * LEN;
            const char* p = (const char*)target + ((b * (G + 1) + j) * V + v0) * ES;
            warp_ring_load(r, k, p, (uint32_t)(min((int64_t)LEN, V - v0) * ES), Ch::NEG_INF_WORD);
            ++issued[s];
        }
    };
    using Slot0 = std::integral_constant<int, 0>;
    using Slot1 = std::integral_constant<int, 1>;
    // unit k in slot S_: reduce it (unless skipped), refill the slot with unit
    // k + 2, count the unit; false if a copy never arrived
    auto step = [&](auto S_, int k) -> bool {
        constexpr int s = decltype(S_)::value;
        const int64_t b = sb[s];
        const int j = sj[s], c = sc[s];
        // the skip word of unit k + 2's sequence, read now and used after this
        // unit's work, so its latency is hidden
        unsigned seen = 0u;
        if (k + 2 < n) {
            int64_t b2;
            int j2, c2;
            unit_of(k + 2, b2, j2, c2);
            seen = *(volatile unsigned*)&skipw[b2];
        }
        if (!skip[s]) {
            if (!mbar_wait(r.bar + 8 * s, (issued[s] - 1u) & 1u)) {
                if (lane == 0) {  // the copies still in flight land before the CTA may exit
                    atomicOr(&g_dev_err, ERR_STREAM);
                    if (!skip[0]) mbar_wait(r.bar, (issued[0] - 1u) & 1u);
                    if (!skip[1]) mbar_wait(r.bar + 8, (issued[1] - 1u) & 1u);
                }
                return false;
            }
            const int64_t v0 = (int64_t)c * LEN;
            const uint64_t key =
                greedy_chunk<BF16>(SmemView<BF16>{r.slot(k), v0, (int)min((int64_t)LEN, V - v0)});
            r.done(k);
            if (lane == 0) {
                part[(b * (G + 1) + j) * S + c] = key;
                if (j < G && key > dkey[s]) {
                    atomicMax(&skipw[b], (unsigned)(G + 1 - j));
                    atomicMax(&s_skip[b], (unsigned)(G + 1 - j));
                }
            }
        }
        if (k + 2 < n) bring(S_, k + 2, seen);
        bool last = false;
        if (lane == 0) last = publish(&counters[b], 1u, (unsigned)((G + 1) * S));
        if (__shfl_sync(FULL, last, 0)) {
            __syncwarp();  // lane 0's acquire covers the whole warp's reads
            greedy_finish(part + b * (G + 1) * S, S, G, V, (int)b, draft_tok, n_accept, out_tok);
            if (lane == 0) {  // every unit of the sequence is counted: leave its words zero
                counters[b] = 0u;
                skipw[b] = 0u;
            }
        }
        return true;
    };
    if (n > 0) bring(Slot0{}, 0, 0u);
    if (n > 1) bring(Slot1{}, 1, 0u);
    for (int k = 0; k < n; k += 2) {
        if (!step(Slot0{}, k)) return;
        if (k + 1 < n && !step(Slot1{}, k + 1)) return;
    }
}

}  // namespace dfl

using namespace dfl;
using namespace dfl_host;

extern "C" int dflash2_verify_greedy(const void* target, int dtype, int B, int G, int64_t V,
                                     const int32_t* draft_tok, int32_t* n_accept, int32_t* out_tok,
                                     void* ws, size_t ws_bytes, dflash2_stream_t stream);

extern "C" int dflash2_verify_greedy_early_exit(const void* target, int dtype, int B, int G,
                                                int64_t V, const int32_t* draft_tok,
                                                int32_t* n_accept, int32_t* out_tok, void* ws,
                                                size_t ws_bytes, dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (B < 0 || G < 1 || G >= DFLASH2_MAX_BLOCK || V < 1 || V > INT32_MAX) return DFLASH2_ESHAPE;
    if (B == 0) return DFLASH2_OK;
    if (!target || !draft_tok || !n_accept || !out_tok) return DFLASH2_EINVAL;
    const int es = elem_size(dtype);
    if (!aligned(target, es) || !aligned(draft_tok, 4) || !aligned(n_accept, 4) ||
        !aligned(out_tok, 4))
        return DFLASH2_EALIGN;
    // rows that TMA cannot copy in whole chunks, or more drafted tokens than
    // the kernel's shared tables hold: the full verify (same results)
    if (!aligned(target, 16) || (V * es) % 16 != 0 || (int64_t)B * G > EE_MAX_TOK ||
        B > EE_MAX_SEQ)
        return dflash2_verify_greedy(target, dtype, B, G, V, draft_tok, n_accept, out_tok, ws,
                                     ws_bytes, stream);
    const int64_t S = row_chunks(V, es);
    const int64_t units = (int64_t)B * (G + 1) * S;
    if (units > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = greedy_ee_layout(B, G, V, es);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    unsigned* skipw = counters + B;
    uint64_t* part = (uint64_t*)((char*)ws + L.part_off);
    if (!L.self_clean && cudaMemsetAsync(counters, 0, (size_t)B * 8, s) != cudaSuccess)
        return DFLASH2_ECUDA;
#define DFL_GEE(BF)                                                                              \
    do {                                                                                         \
        auto kern = verify_greedy_ee_kernel<BF>;                                                 \
        if (ring_prepare(kern, RING_BYTES) != DFLASH2_OK) return DFLASH2_ECUDA;                  \
        kern<<<ring_grid(units), RING_THREADS, RING_BYTES, s>>>(target, B, G, V, (int)S, units,  \
                                                                draft_tok, n_accept, out_tok,   \
                                                                part, counters, skipw);         \
    } while (0)
    if (dtype == DFLASH2_BF16) DFL_GEE(true);
    else DFL_GEE(false);
#undef DFL_GEE
    return launch_status();
}

unsigned dfl_errors_greedy_ee(int clear) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_err, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (clear && v) {
        unsigned z = 0;
        cudaMemcpyToSymbol(g_dev_err, &z, sizeof z);
    }
    return v;
}
