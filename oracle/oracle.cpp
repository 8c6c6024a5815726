/*
 * Oracle for the simulated-communicator collectives: a plain, slow, obviously correct CPU
 * implementation of what every collective computes.
 *
 * THIS IS TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * load it. It shares no code, header, table or helper with the CUDA library, and the CUDA library
 * never calls it. Each function follows the passage cited above it.
 *
 * Pages cited:
 *   [Atlas]  "集合通信：原语、算法、NCCL 实现与拓扑映射" (llm-infra-atlas.github.io/hpc/04_collectives)
 *   [Primer] "Collective Communication：AllReduce、AllGather、ReduceScatter 与 All-to-All"
 *            (charlestar.github.io/2026/08/20/gpu-collective-communication)
 *   [Eight]  "详解分布式训练8大集合通信原语：从Send/Recv到All2All" (bjdmk.com.cn/news/4699717)
 *
 * Conventions (our own; the pages write the data layouts only as figures):
 *   - p ranks; rank r's buffer is in[r] / out[r], a host pointer.
 *   - n is the per-rank full-buffer element count: the AllReduce in/out size, the ReduceScatter
 *     input size, the AllGather output size and the All-to-All send size ([Primer] section
 *     "先统一通信量的记号", where B is the full logical tensor).
 *   - dtype 0 = int32, 1 = fp32, 2 = bf16 (stored as the upper 16 bits of an IEEE fp32).
 *   - op 0 = sum, 1 = min, 2 = max, 3 = avg (sum times 1/p).
 *   - acc 0 = EXACT: sums in double in rank order, rounded once to the output type.
 *     acc 1 = RANKFOLD: the fp32 left fold acc = x0; acc = acc + x1; ... in rank order (for the
 *     MoE combine, the same fold over a token's slots; see that section).
 *
 * Return value: 0 on success, -1 on an argument the definitions do not cover; the MoE dispatch
 * also returns 1 when a destination's capacity is too small.
 *
 * Parity pins: every function here is pinned by a CPU test against the pages' worked example,
 * figure layouts, hand-derived small examples, identities, closed forms or brute force, and a
 * mutation test plants plausible mistakes in a copy of this file and checks that a pin fails. The ring schedule itself (as opposed to
 * its result) is "parity unpinned": the page's p = 4 trace is garbled, so the schedule follows the
 * reading that makes rank r own block r.
 */
#include <algorithm>
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

enum { DT_INT32 = 0, DT_FP32 = 1, DT_BF16 = 2 };
enum { OP_SUM = 0, OP_MIN = 1, OP_MAX = 2, OP_AVG = 3 };
enum { ACC_EXACT = 0, ACC_RANKFOLD = 1 };

size_t elem_size(int dtype) { return dtype == DT_BF16 ? 2 : 4; }

bool valid_dtype(int dtype) { return dtype == DT_INT32 || dtype == DT_FP32 || dtype == DT_BF16; }

/* ---- IEEE conversions written from the definitions -------------------------------------------- */

float bits_to_float(uint32_t u) {
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

uint32_t float_to_bits(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return u;
}

/* A bf16 value is the top half of an fp32 bit pattern. */
float bf16_to_float(uint16_t h) { return bits_to_float(uint32_t(h) << 16); }

/* fp32 -> bf16, round to nearest, ties to even, on the 16 dropped bits. NaN stays NaN. */
uint16_t float_to_bf16_rne(float f) {
    uint32_t u = float_to_bits(f);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0) return uint16_t((u >> 16) | 0x40);
    uint32_t lower = u & 0xFFFFu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;  // carry may reach inf: correct
    return uint16_t(upper);
}

/* double -> bf16 with a single rounding (no detour through fp32): round |x| to the bf16 grid
 * (8 significant bits for normal numbers, spacing 2^-133 below 2^-126), ties to even. */
uint16_t double_to_bf16_rne(double x) {
    if (std::isnan(x)) return 0x7FC0;
    bool neg = std::signbit(x);
    double a = std::fabs(x);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else {
        int e;
        std::frexp(a, &e);                 // a = m * 2^e, m in [0.5, 1)
        int q = e - 8;                     // 8 significant bits -> quantum 2^(e-8)
        if (q < -133) q = -133;            // subnormal spacing
        double scaled = std::ldexp(a, -q);
        double rounded = std::nearbyint(scaled);  // default rounding mode: ties to even
        r = std::ldexp(rounded, q);
    }
    float f = float(r);                    // exact: r has at most 8 significant bits, or overflows to inf
    if (r >= 0x1p128) f = INFINITY;
    uint16_t h = uint16_t(float_to_bits(f) >> 16);
    return neg ? uint16_t(h | 0x8000u) : h;
}

/* ---- element access ---------------------------------------------------------------------------- */

double load_as_double(const void* buf, int dtype, size_t i) {
    if (dtype == DT_INT32) return double(static_cast<const int32_t*>(buf)[i]);
    if (dtype == DT_FP32) return double(static_cast<const float*>(buf)[i]);
    return double(bf16_to_float(static_cast<const uint16_t*>(buf)[i]));
}

float load_as_float(const void* buf, int dtype, size_t i) {
    if (dtype == DT_FP32) return static_cast<const float*>(buf)[i];
    return bf16_to_float(static_cast<const uint16_t*>(buf)[i]);
}

void store_float(void* buf, int dtype, size_t i, float v) {
    if (dtype == DT_FP32)
        static_cast<float*>(buf)[i] = v;
    else
        static_cast<uint16_t*>(buf)[i] = float_to_bf16_rne(v);
}

void store_double_rounded_once(void* buf, int dtype, size_t i, double v) {
    if (dtype == DT_FP32)
        static_cast<float*>(buf)[i] = float(v);  // C conversion rounds to nearest even
    else
        static_cast<uint16_t*>(buf)[i] = double_to_bf16_rne(v);
}

void copy_element(const void* src, size_t si, void* dst, size_t di, int dtype) {
    size_t d = elem_size(dtype);
    std::memcpy(static_cast<char*>(dst) + di * d, static_cast<const char*>(src) + si * d, d);
}

/* ---- the reduction operator ⊕ ----------------------------------------------------------------- */

/* min/max as a left fold: the earlier operand is kept on ties. */
template <typename T>
T apply_minmax(int op, T a, T b) {
    if (op == OP_MIN) return (b < a) ? b : a;
    return (a < b) ? b : a;
}

/* Reduce element i over the given rank order and store it to out at index oi.
 * [Atlas] §1.3/§1.4: out[i] = in_0[i] ⊕ in_1[i] ⊕ ... ⊕ in_{p-1}[i] (⊕ = sum, min or max).
 * AVG is sum times 1/p: [Atlas] §1.4 notes that DDP takes the mean as a sum followed by a division
 * by the world size. */
void reduce_element(int p, const void* const* in, const std::vector<int>& order, size_t i, int dtype,
                    int op, int acc, void* out, size_t oi) {
    if (dtype == DT_INT32) {
        const int32_t* first = static_cast<const int32_t*>(in[order[0]]);
        if (op == OP_SUM) {
            uint32_t s = uint32_t(first[i]);  // two's-complement wraparound
            for (int k = 1; k < p; ++k) s += uint32_t(static_cast<const int32_t*>(in[order[k]])[i]);
            static_cast<int32_t*>(out)[oi] = int32_t(s);
        } else {
            int32_t v = first[i];
            for (int k = 1; k < p; ++k) v = apply_minmax(op, v, static_cast<const int32_t*>(in[order[k]])[i]);
            static_cast<int32_t*>(out)[oi] = v;
        }
        return;
    }
    if (op == OP_MIN || op == OP_MAX) {
        float v = load_as_float(in[order[0]], dtype, i);
        for (int k = 1; k < p; ++k) v = apply_minmax(op, v, load_as_float(in[order[k]], dtype, i));
        store_float(out, dtype, oi, v);  // v is one of the inputs: exact in any precision
        return;
    }
    if (acc == ACC_EXACT) {
        double s = load_as_double(in[order[0]], dtype, i);
        for (int k = 1; k < p; ++k) s += load_as_double(in[order[k]], dtype, i);
        if (op == OP_AVG) s = s / double(p);
        store_double_rounded_once(out, dtype, oi, s);
    } else {
        volatile float s = load_as_float(in[order[0]], dtype, i);
        for (int k = 1; k < p; ++k) s = s + load_as_float(in[order[k]], dtype, i);
        float v = s;
        if (op == OP_AVG) {
            volatile float scale = 1.0f / float(p);
            v = v * scale;
        }
        store_float(out, dtype, oi, v);
    }
}

bool valid_common(int p, int dtype) { return p >= 1 && valid_dtype(dtype); }

bool valid_reduce_args(int p, int dtype, int op, int acc) {
    if (!valid_common(p, dtype)) return false;
    if (op < OP_SUM || op > OP_AVG) return false;
    if (dtype == DT_INT32 && op == OP_AVG) return false;
    return acc == ACC_EXACT || acc == ACC_RANKFOLD;
}

std::vector<int> rank_order(int p) {
    std::vector<int> o(p);
    for (int r = 0; r < p; ++r) o[r] = r;
    return o;
}

int mod(long long a, int p) { return int(((a % p) + p) % p); }

/* Ring segment k of an n-element buffer: p equal chunks of ceil(n/p) elements, the last ones
 * shorter (possibly empty). [Primer] "Ring AllReduce 怎样拆成两半" assumes B splits evenly into
 * p chunks; when it does, this is exactly that split. */
void ring_segment(size_t n, int p, int k, size_t* begin, size_t* end) {
    size_t seg = (n + size_t(p) - 1) / size_t(p);
    size_t b = size_t(k) * seg, e = b + seg;
    if (b > n) b = n;
    if (e > n) e = n;
    *begin = b;
    *end = e;
}

/* Accumulator of the ring emulation: fp32 for fp32/bf16, wrapping uint32 for int32 sums, the
 * exact int32 for int32 min/max. */
struct RingAcc {
    int dtype, op;
    std::vector<float> f;
    std::vector<int32_t> i;
    void resize(size_t n) {
        if (dtype == DT_INT32) i.assign(n, 0); else f.assign(n, 0.0f);
    }
    void load(const void* src, size_t k) {
        if (dtype == DT_INT32) i[k] = static_cast<const int32_t*>(src)[k];
        else f[k] = load_as_float(src, dtype, k);
    }
    /* this[k] = received ⊕ own, received first (it carries the earlier ranks of the chain). */
    void combine(float received_f, int32_t received_i, const void* own, size_t k) {
        if (dtype == DT_INT32) {
            int32_t o = static_cast<const int32_t*>(own)[k];
            if (op == OP_SUM) i[k] = int32_t(uint32_t(received_i) + uint32_t(o));
            else i[k] = apply_minmax(op, received_i, o);
        } else {
            volatile float r = received_f;
            float o = load_as_float(own, dtype, k);
            if (op == OP_MIN || op == OP_MAX) f[k] = apply_minmax(op, float(r), o);
            else { volatile float s = r + o; f[k] = s; }
        }
    }
    /* Final value of a fully reduced element: AVG scales in fp32, then one rounding to dtype. */
    void store_final(int p, void* out, size_t oi, size_t k) const {
        if (dtype == DT_INT32) { static_cast<int32_t*>(out)[oi] = i[k]; return; }
        float v = f[k];
        if (op == OP_AVG) { volatile float scale = 1.0f / float(p); v = v * scale; }
        store_float(out, dtype, oi, v);
    }
};

}  // namespace

extern "C" {

/* ===================== plain definitions ======================================================= */

/* [Atlas] §1.4 AllReduce: out_r[i] = ⊕_{r'} in_{r'}[i], identical on every rank r.
 * [Primer] "AllReduce：Partial 变成 Replicated". */
int oracle_allreduce(int p, const void* const* in, void* const* out, size_t n, int dtype, int op, int acc) {
    if (!valid_reduce_args(p, dtype, op, acc)) return -1;
    std::vector<int> order = rank_order(p);
    std::vector<char> tmp(elem_size(dtype));
    for (size_t i = 0; i < n; ++i) {
        reduce_element(p, in, order, i, dtype, op, acc, tmp.data(), 0);
        for (int r = 0; r < p; ++r) copy_element(tmp.data(), 0, out[r], i, dtype);
    }
    return 0;
}

/* [Atlas] §1.3 Reduce: out_root[i] = ⊕_r in_r[i]; only the root's buffer receives it (the other
 * ranks' outputs are shown empty and are left untouched here). Root is a rank index ([Atlas] §0). */
int oracle_reduce(int p, const void* const* in, void* out_root, size_t n, int dtype, int op, int root, int acc) {
    if (!valid_reduce_args(p, dtype, op, acc) || root < 0 || root >= p) return -1;
    std::vector<int> order = rank_order(p);
    for (size_t i = 0; i < n; ++i) reduce_element(p, in, order, i, dtype, op, acc, out_root, i);
    return 0;
}

/* [Atlas] §1.1 Broadcast: the root's n-element buffer is copied to every rank, root included. */
int oracle_broadcast(int p, const void* in_root, void* const* out, size_t n, int dtype, int root) {
    if (!valid_common(p, dtype) || root < 0 || root >= p) return -1;
    for (int r = 0; r < p; ++r)
        for (size_t i = 0; i < n; ++i) copy_element(in_root, i, out[r], i, dtype);
    return 0;
}

/* [Atlas] §1.5 ReduceScatter: each rank holds [p·m] (m = n/p); the reduction of block r goes to
 * rank r: out_r[k] = ⊕_q in_q[r·m + k]. */
int oracle_reduce_scatter(int p, const void* const* in, void* const* out, size_t n, int dtype, int op, int acc) {
    if (!valid_reduce_args(p, dtype, op, acc) || n % size_t(p) != 0) return -1;
    size_t m = n / size_t(p);
    std::vector<int> order = rank_order(p);
    for (int r = 0; r < p; ++r)
        for (size_t k = 0; k < m; ++k) reduce_element(p, in, order, size_t(r) * m + k, dtype, op, acc, out[r], k);
    return 0;
}

/* [Atlas] §1.2 AllGather: p shards of m = n/p elements are concatenated in rank order and every
 * rank receives the [p·m] result: out_r[q·m + k] = in_q[k]. */
int oracle_allgather(int p, const void* const* in, void* const* out, size_t n, int dtype) {
    if (!valid_common(p, dtype) || n % size_t(p) != 0) return -1;
    size_t m = n / size_t(p);
    for (int r = 0; r < p; ++r)
        for (int q = 0; q < p; ++q)
            for (size_t k = 0; k < m; ++k) copy_element(in[q], k, out[r], size_t(q) * m + k, dtype);
    return 0;
}

/* [Atlas] §1.6 AllToAll: the [src][dst] block matrix is transposed. Block j of source i lands as
 * block i of destination j: out_j[i·m + k] = in_i[j·m + k], m = n/p. */
int oracle_alltoall(int p, const void* const* in, void* const* out, size_t n, int dtype) {
    if (!valid_common(p, dtype) || n % size_t(p) != 0) return -1;
    size_t m = n / size_t(p);
    for (int i = 0; i < p; ++i)
        for (int j = 0; j < p; ++j)
            for (size_t k = 0; k < m; ++k) copy_element(in[i], size_t(j) * m + k, out[j], size_t(i) * m + k, dtype);
    return 0;
}

/* [Primer] "Ragged All-to-All：MoE 的真实输入通常不等长": c_ij elements go from source i to
 * destination j; counts -> prefix-sum offsets -> payload exchange. Source i packs its blocks in
 * destination order, destination j stores them in source order:
 *   sdispl_i[j] = Σ_{j'<j} c_ij',  rdispl_j[i] = Σ_{i'<i} c_i'j,
 *   out_j[rdispl_j[i] + k] = in_i[sdispl_i[j] + k] for k < c_ij.
 * counts is row-major [p][p]; recv_counts (may be null) gets Σ_i c_ij per destination j.
 * Negative counts are outside the definition. */
int oracle_alltoallv(int p, const void* const* in, void* const* out, const int64_t* counts, int dtype,
                     int64_t* recv_counts) {
    if (!valid_common(p, dtype)) return -1;
    for (int a = 0; a < p * p; ++a)
        if (counts[a] < 0) return -1;
    for (int i = 0; i < p; ++i) {
        for (int j = 0; j < p; ++j) {
            int64_t sdispl = 0;
            for (int jj = 0; jj < j; ++jj) sdispl += counts[i * p + jj];
            int64_t rdispl = 0;
            for (int ii = 0; ii < i; ++ii) rdispl += counts[ii * p + j];
            for (int64_t k = 0; k < counts[i * p + j]; ++k)
                copy_element(in[i], size_t(sdispl + k), out[j], size_t(rdispl + k), dtype);
        }
    }
    if (recv_counts) {
        for (int j = 0; j < p; ++j) {
            int64_t s = 0;
            for (int i = 0; i < p; ++i) s += counts[i * p + j];
            recv_counts[j] = s;
        }
    }
    return 0;
}

/* [Eight] "3.3 Scatter": the root's data is cut into p blocks in rank order and block r goes to
 * rank r ([Atlas] §0 lists Gather/Scatter as the single-root forms): out_r[k] = in_root[r·m + k],
 * m = n/p. Only the root's input is read. */
int oracle_scatter(int p, const void* in_root, void* const* out, size_t n, int dtype, int root) {
    if (!valid_common(p, dtype) || root < 0 || root >= p || n % size_t(p) != 0) return -1;
    size_t m = n / size_t(p);
    for (int r = 0; r < p; ++r)
        for (size_t k = 0; k < m; ++k) copy_element(in_root, size_t(r) * m + k, out[r], k, dtype);
    return 0;
}

/* [Eight] "4.3 Gather": every rank's block is collected at the root only, in rank order:
 * out_root[r·m + k] = in_r[k], m = n/p. Only the root's output is written. */
int oracle_gather(int p, const void* const* in, void* out_root, size_t n, int dtype, int root) {
    if (!valid_common(p, dtype) || root < 0 || root >= p || n % size_t(p) != 0) return -1;
    size_t m = n / size_t(p);
    for (int r = 0; r < p; ++r)
        for (size_t k = 0; k < m; ++k) copy_element(in[r], k, out_root, size_t(r) * m + k, dtype);
    return 0;
}

/* ===================== ring schedule emulation ================================================== */
/* [Atlas] §2.2: ranks form the ring r0 -> r1 -> ... -> r_{p-1} -> r0, every buffer is cut into p
 * chunks, a ring reduce-scatter of p-1 steps is followed by a ring all-gather of p-1 steps.
 * Reading of the page's garbled p = 4 trace: at reduce-scatter step s (1..p-1) rank r sends its
 * current chunk (r - s) mod p to rank r+1, which adds its own input to it; after step p-1 rank r
 * holds the fully reduced chunk r, matching ReduceScatter's owner rule ([Atlas] §1.5). At
 * all-gather step s (1..p-1) rank r forwards chunk (r - s + 1) mod p to rank r+1. The partials
 * travel in fp32 for fp32 and bf16 data; an owner rounds once when its chunk is complete. */

static int ring_reduce_scatter_phase(int p, const void* const* in, size_t n, int dtype, int op,
                                     std::vector<RingAcc>& part) {
    part.assign(p, RingAcc{dtype, op, {}, {}});
    for (int r = 0; r < p; ++r) part[r].resize(n);
    /* Step 1 sends raw inputs: seed every rank's partial with its own input. */
    for (int r = 0; r < p; ++r)
        for (size_t k = 0; k < n; ++k) part[r].load(in[r], k);
    /* The receiver's partial of a chunk it has not reduced yet is its raw input, so "receive and
     * add" overwrites the chunk with received ⊕ own. */
    for (int s = 1; s <= p - 1; ++s) {
        /* messages of this step: rank r sends chunk (r - s) mod p to rank r+1 */
        std::vector<std::vector<float>> msg_f(p);
        std::vector<std::vector<int32_t>> msg_i(p);
        std::vector<int> msg_chunk(p);
        for (int r = 0; r < p; ++r) {
            int c = mod(r - s, p);
            size_t b, e;
            ring_segment(n, p, c, &b, &e);
            int dst = mod(r + 1, p);
            msg_chunk[dst] = c;
            if (dtype == DT_INT32) msg_i[dst].assign(part[r].i.begin() + b, part[r].i.begin() + e);
            else msg_f[dst].assign(part[r].f.begin() + b, part[r].f.begin() + e);
        }
        for (int q = 0; q < p; ++q) {
            int c = msg_chunk[q];
            size_t b, e;
            ring_segment(n, p, c, &b, &e);
            for (size_t k = b; k < e; ++k)
                part[q].combine(dtype == DT_INT32 ? 0.0f : msg_f[q][k - b], dtype == DT_INT32 ? msg_i[q][k - b] : 0,
                                in[q], k);
        }
    }
    return 0;
}

/* Ring AllReduce = ring ReduceScatter then ring AllGather ([Atlas] §0 second identity, §2.2). */
int oracle_ring_allreduce(int p, const void* const* in, void* const* out, size_t n, int dtype, int op) {
    if (!valid_reduce_args(p, dtype, op, ACC_RANKFOLD)) return -1;
    std::vector<RingAcc> part;
    ring_reduce_scatter_phase(p, in, n, dtype, op, part);
    /* owners round their complete chunk into their own output */
    for (int r = 0; r < p; ++r) {
        size_t b, e;
        ring_segment(n, p, r, &b, &e);
        for (size_t k = b; k < e; ++k) part[r].store_final(p, out[r], k, k);
    }
    /* all-gather: step s, rank r forwards chunk (r - s + 1) mod p of its output to rank r+1 */
    size_t d = elem_size(dtype);
    for (int s = 1; s <= p - 1; ++s) {
        std::vector<std::vector<char>> msg(p);
        std::vector<int> msg_chunk(p);
        for (int r = 0; r < p; ++r) {
            int c = mod(r - s + 1, p);
            size_t b, e;
            ring_segment(n, p, c, &b, &e);
            int dst = mod(r + 1, p);
            msg_chunk[dst] = c;
            const char* src = static_cast<const char*>(out[r]);
            msg[dst].assign(src + b * d, src + e * d);
        }
        for (int q = 0; q < p; ++q) {
            size_t b, e;
            ring_segment(n, p, msg_chunk[q], &b, &e);
            if (e > b) std::memcpy(static_cast<char*>(out[q]) + b * d, msg[q].data(), (e - b) * d);
        }
    }
    return 0;
}

/* Ring ReduceScatter: the reduce-scatter phase alone; rank r outputs its complete chunk r. */
int oracle_ring_reduce_scatter(int p, const void* const* in, void* const* out, size_t n, int dtype, int op) {
    if (!valid_reduce_args(p, dtype, op, ACC_RANKFOLD) || n % size_t(p) != 0) return -1;
    std::vector<RingAcc> part;
    ring_reduce_scatter_phase(p, in, n, dtype, op, part);
    size_t m = n / size_t(p);
    for (int r = 0; r < p; ++r)
        for (size_t k = 0; k < m; ++k) part[r].store_final(p, out[r], k, size_t(r) * m + k);
    return 0;
}

/* Ring AllGather: rank r starts with its shard as chunk r of its output; at step s it forwards
 * chunk (r - s + 1) mod p to rank r+1. n is the output element count (m = n/p per shard). */
int oracle_ring_allgather(int p, const void* const* in, void* const* out, size_t n, int dtype) {
    if (!valid_common(p, dtype) || n % size_t(p) != 0) return -1;
    size_t m = n / size_t(p), d = elem_size(dtype);
    for (int r = 0; r < p; ++r)
        if (m) std::memcpy(static_cast<char*>(out[r]) + size_t(r) * m * d, in[r], m * d);
    for (int s = 1; s <= p - 1; ++s) {
        std::vector<std::vector<char>> msg(p);
        std::vector<int> msg_chunk(p);
        for (int r = 0; r < p; ++r) {
            int c = mod(r - s + 1, p);
            int dst = mod(r + 1, p);
            msg_chunk[dst] = c;
            const char* src = static_cast<const char*>(out[r]) + size_t(c) * m * d;
            msg[dst].assign(src, src + m * d);
        }
        for (int q = 0; q < p; ++q)
            if (m) std::memcpy(static_cast<char*>(out[q]) + size_t(msg_chunk[q]) * m * d, msg[q].data(), m * d);
    }
    return 0;
}

/* Ring Reduce (our reading: the pages define rings only for AllReduce/ReduceScatter/AllGather):
 * a chain root+1 -> root+2 -> ... -> root. The first rank sends its raw input, each next rank adds
 * its own input to what it received, the root rounds the complete result. */
int oracle_ring_reduce(int p, const void* const* in, void* out_root, size_t n, int dtype, int op, int root) {
    if (!valid_reduce_args(p, dtype, op, ACC_RANKFOLD) || root < 0 || root >= p) return -1;
    RingAcc held{dtype, op, {}, {}};
    held.resize(n);
    int first = mod(root + 1, p);
    for (size_t k = 0; k < n; ++k) held.load(in[first], k);
    for (int h = 1; h <= p - 1; ++h) {
        int q = mod(root + 1 + h, p);
        RingAcc received = held;  // the message from the previous rank of the chain
        for (size_t k = 0; k < n; ++k)
            held.combine(dtype == DT_INT32 ? 0.0f : received.f[k], dtype == DT_INT32 ? received.i[k] : 0, in[q], k);
    }
    for (size_t k = 0; k < n; ++k) held.store_final(p, out_root, k, k);
    return 0;
}

/* Ring Broadcast (our reading): a chain root -> root+1 -> ... -> root-1 of p-1 hops; the root's
 * own output receives the root's input too. */
int oracle_ring_broadcast(int p, const void* in_root, void* const* out, size_t n, int dtype, int root) {
    if (!valid_common(p, dtype) || root < 0 || root >= p) return -1;
    size_t d = elem_size(dtype);
    if (n) std::memcpy(out[root], in_root, n * d);
    for (int h = 1; h <= p - 1; ++h) {
        int src = mod(root + h - 1, p), dst = mod(root + h, p);
        if (n) std::memcpy(out[dst], out[src], n * d);
    }
    return 0;
}

/* Ring All-to-All (our reading): the p-1 step shift exchange. Step 0 keeps the own block; at step s
 * rank r sends its block (r+s) mod p to rank (r+s) mod p. */
int oracle_ring_alltoall(int p, const void* const* in, void* const* out, size_t n, int dtype) {
    if (!valid_common(p, dtype) || n % size_t(p) != 0) return -1;
    size_t m = n / size_t(p), d = elem_size(dtype);
    for (int s = 0; s <= p - 1; ++s)
        for (int r = 0; r < p; ++r) {
            int j = mod(r + s, p);
            if (m)
                std::memcpy(static_cast<char*>(out[j]) + size_t(r) * m * d,
                            static_cast<const char*>(in[r]) + size_t(j) * m * d, m * d);
        }
    return 0;
}

/* ===================== recursive doubling / halving-doubling ====================================== */
/* [Atlas] §2.3 (p a power of two). Reading (the page gives the exchange pattern, not the operand
 * order): when partners r and r^d combine, the lower rank's data comes first, so both compute the
 * same value; partials travel in fp32 for fp32 and bf16 data and are rounded once at the end. */

static bool power_of_two(int p) { return p >= 1 && (p & (p - 1)) == 0; }

/* Recursive doubling: at step k (distance d = 2^k) every rank replaces its vector by
 * vec[min(r, r^d)] ⊕ vec[max(r, r^d)]; after log2(p) steps every rank holds the reduction. */
int oracle_rd_allreduce(int p, const void* const* in, void* const* out, size_t n, int dtype, int op) {
    if (!valid_reduce_args(p, dtype, op, ACC_RANKFOLD) || !power_of_two(p)) return -1;
    std::vector<RingAcc> cur(p, RingAcc{dtype, op, {}, {}});
    for (int r = 0; r < p; ++r) {
        cur[r].resize(n);
        for (size_t k = 0; k < n; ++k) cur[r].load(in[r], k);
    }
    for (int d = 1; d < p; d <<= 1) {
        std::vector<RingAcc> next = cur;  // every rank reads the values of the previous step
        for (int r = 0; r < p; ++r) {
            const int lo = std::min(r, r ^ d), hi = std::max(r, r ^ d);
            for (size_t k = 0; k < n; ++k) {
                if (dtype == DT_INT32) {
                    int32_t a = cur[lo].i[k], b = cur[hi].i[k];
                    next[r].i[k] = (op == OP_SUM) ? int32_t(uint32_t(a) + uint32_t(b)) : apply_minmax(op, a, b);
                } else {
                    volatile float a = cur[lo].f[k], b = cur[hi].f[k];
                    if (op == OP_MIN || op == OP_MAX) next[r].f[k] = apply_minmax(op, float(a), float(b));
                    else { volatile float sum = a + b; next[r].f[k] = sum; }
                }
            }
        }
        cur.swap(next);
    }
    for (int r = 0; r < p; ++r)
        for (size_t k = 0; k < n; ++k) cur[r].store_final(p, out[r], k, k);
    return 0;
}

/* Recursive halving-doubling (reduce-scatter by halving, then all-gather by doubling). The buffer
 * is cut into p blocks as in the ring (ring_segment). Halving step with distance d = p/2, p/4, ..., 1:
 * rank r's blocks are the aligned group of 2d blocks containing block r; it keeps the half that
 * contains block r and computes kept = mine ⊕ partner's (lower rank first) while the partner keeps
 * the other half. After the last step rank r holds the complete block r. Doubling steps with
 * d = 1, 2, ..., p/2: partners exchange the groups of d blocks they hold. */
int oracle_hd_allreduce(int p, const void* const* in, void* const* out, size_t n, int dtype, int op) {
    if (!valid_reduce_args(p, dtype, op, ACC_RANKFOLD) || !power_of_two(p)) return -1;
    std::vector<RingAcc> cur(p, RingAcc{dtype, op, {}, {}});
    for (int r = 0; r < p; ++r) {
        cur[r].resize(n);
        for (size_t k = 0; k < n; ++k) cur[r].load(in[r], k);
    }
    for (int d = p / 2; d >= 1; d >>= 1) {
        std::vector<RingAcc> next = cur;
        for (int r = 0; r < p; ++r) {
            const int partner = r ^ d, lo = std::min(r, partner), hi = std::max(r, partner);
            const int group = (r / (2 * d)) * (2 * d);
            const int kb = (r & d) ? group + d : group;  // first block of the kept half
            size_t b0, e0, b1, e1;
            ring_segment(n, p, kb, &b0, &e0);
            ring_segment(n, p, kb + d - 1, &b1, &e1);
            for (size_t k = b0; k < e1; ++k) {
                if (dtype == DT_INT32) {
                    int32_t a = cur[lo].i[k], b = cur[hi].i[k];
                    next[r].i[k] = (op == OP_SUM) ? int32_t(uint32_t(a) + uint32_t(b)) : apply_minmax(op, a, b);
                } else {
                    volatile float a = cur[lo].f[k], b = cur[hi].f[k];
                    if (op == OP_MIN || op == OP_MAX) next[r].f[k] = apply_minmax(op, float(a), float(b));
                    else { volatile float sum = a + b; next[r].f[k] = sum; }
                }
            }
        }
        cur.swap(next);
    }
    /* rank r rounds its complete block r; then the doubling exchanges spread the blocks */
    for (int r = 0; r < p; ++r) {
        size_t b, e;
        ring_segment(n, p, r, &b, &e);
        for (size_t k = b; k < e; ++k) cur[r].store_final(p, out[r], k, k);
    }
    size_t dsz = elem_size(dtype);
    for (int d = 1; d < p; d <<= 1) {
        std::vector<std::vector<char>> snapshot(p);
        for (int r = 0; r < p; ++r) {
            const char* o = static_cast<const char*>(out[r]);
            snapshot[r].assign(o, o + n * dsz);
        }
        for (int r = 0; r < p; ++r) {
            const int partner = r ^ d;
            const int pg = (partner / d) * d;  // the partner's group of d blocks
            size_t b0, e0, b1, e1;
            ring_segment(n, p, pg, &b0, &e0);
            ring_segment(n, p, pg + d - 1, &b1, &e1);
            if (e1 > b0)
                std::memcpy(static_cast<char*>(out[r]) + b0 * dsz, snapshot[partner].data() + b0 * dsz, (e1 - b0) * dsz);
        }
    }
    return 0;
}

/* ===================== tree AllReduce ============================================================ */
/* [Primer] "Tree AllReduce 为什么更适合延迟敏感区间": reduce up a tree to its root, then broadcast
 * the result down the same tree, in a number of rounds logarithmic in p. [Atlas] §2.4 "double
 * binary tree": two complementary binary trees over the same ranks, drawn as tree A = 0 -> {1, 2},
 * 1 -> {3, 4}, 2 -> {5, 6} and tree B = the same shape with rank p-1-m where tree A has rank m.
 * Readings (ours): a tree is the heap numbering of positions m = 0..p-1 (children 2m+1 and 2m+2
 * when < p, the root at position 0); tree A puts rank m at position m, tree B rank p-1-m. A
 * position's partial is its rank's input ⊕ its left child's partial ⊕ its right child's partial,
 * folded in that order, in fp32 for fp32/bf16 data (wrapping int32 for int32 sums); the root's
 * value is scaled for AVG, rounded once and passed down unchanged. The single tree (double_tree =
 * 0) reduces all n elements on tree A; the double tree (double_tree = 1) reduces elements
 * [0, ceil(n/2)) on tree A and the rest on tree B. */
int oracle_tree_allreduce(int p, const void* const* in, void* const* out, size_t n, int dtype, int op,
                          int double_tree) {
    if (!valid_reduce_args(p, dtype, op, ACC_RANKFOLD) || (double_tree != 0 && double_tree != 1)) return -1;
    const size_t half = double_tree ? (n + 1) / 2 : n;
    std::vector<float> f(p);
    std::vector<int32_t> iv(p);
    for (size_t k = 0; k < n; ++k) {
        const bool mirror = k >= half;
        for (int m = p - 1; m >= 0; --m) {  // children sit at larger positions: they are done first
            const int r = mirror ? p - 1 - m : m;
            float af = 0.0f;
            int32_t ai = 0;
            if (dtype == DT_INT32) ai = static_cast<const int32_t*>(in[r])[k];
            else af = load_as_float(in[r], dtype, k);
            for (int c = 2 * m + 1; c <= 2 * m + 2 && c < p; ++c) {
                if (dtype == DT_INT32) {
                    ai = (op == OP_SUM) ? int32_t(uint32_t(ai) + uint32_t(iv[c])) : apply_minmax(op, ai, iv[c]);
                } else if (op == OP_MIN || op == OP_MAX) {
                    af = apply_minmax(op, af, f[c]);
                } else {
                    volatile float s = af + f[c];
                    af = s;
                }
            }
            f[m] = af;
            iv[m] = ai;
        }
        for (int r = 0; r < p; ++r) {
            if (dtype == DT_INT32) {
                static_cast<int32_t*>(out[r])[k] = iv[0];
            } else {
                float v = f[0];
                if (op == OP_AVG) { volatile float scale = 1.0f / float(p); v = v * scale; }
                store_float(out[r], dtype, k, v);
            }
        }
    }
    return 0;
}

/* ===================== MoE dispatch and combine ================================================= */
/* [Primer] "Ragged All-to-All：MoE 的真实输入通常不等长" lists the steps around the variable-split
 * exchange, in this order: router output, counting assignments per destination, exchanging the
 * counts, prefix-summing them into offsets, packing/permuting the payload, the variable-split
 * All-to-All, the experts' compute, the reverse variable-split All-to-All, and unpermute/combine.
 * [Primer] "Expert Parallel：All-to-All 搬运的是 Assignment": the unit that moves is an expert
 * assignment (a token routed to k experts travels k times), and the combine step weights the
 * returning expert outputs with the gate weights and adds the residual, back in source-token layout.
 *
 * Readings (ours; the pages name the steps but not these rules):
 *   - E experts, E a multiple of p; expert e lives on rank e / (E/p);
 *   - the router output of rank i is idx_i[t][s] (token t < T, slot s < k) and, for the combine,
 *     the gate weights w_i[t][s] (fp32);
 *   - pack/permute lists rank i's assignments (t, s) by expert id, ties in token order and then
 *     slot order (a stable sort of the flattened list t*k + s by expert), so every block a
 *     destination receives is grouped by expert;
 *   - the exchange is the Alltoallv above with c_ij = rows from i to j (H elements a row); the
 *     destination layout is [from rank 0 | from rank 1 | ...];
 *   - combine: out_i[t] = residual_i[t] (when given) + Σ_s w_i[t][s] * y_i(t, s), where y_i(t, s)
 *     is the row the expert owner returns for assignment (t, s). acc EXACT sums in double and
 *     rounds once; acc SLOTFOLD (= 1) is the fp32 left fold in slot order (residual first; without
 *     a residual the fold starts at the slot-0 product), every product and sum rounded to fp32.
 * A capacity shortfall (some destination would receive more than cap_rows rows) writes nothing and
 * returns 1; an expert id outside [0, E) is outside the definitions (-1). */

struct MoeRoute {
    int E_loc = 0;
    std::vector<std::vector<int64_t>> cnt;    // [p][E] assignments from rank i to expert e
    std::vector<int64_t> c;                   // [p][p] rows from rank i to rank j
    std::vector<std::vector<int64_t>> order;  // [p][T*k] flattened assignment ids in packed order
};

static int moe_route(int p, const int32_t* const* idx, size_t T, int k, int E, MoeRoute* R) {
    if (p < 1 || k < 1 || E < p || E % p != 0) return -1;
    const size_t A = T * size_t(k);
    R->E_loc = E / p;
    R->cnt.assign(p, std::vector<int64_t>(E, 0));
    R->c.assign(size_t(p) * p, 0);
    R->order.assign(p, std::vector<int64_t>());
    for (int i = 0; i < p; ++i) {
        for (size_t a = 0; a < A; ++a) {  // count assignments per expert, hence per destination
            const int32_t e = idx[i][a];
            if (e < 0 || e >= E) return -1;
            R->cnt[i][e] += 1;
            R->c[size_t(i) * p + e / R->E_loc] += 1;
        }
        std::vector<int64_t>& ord = R->order[i];  // pack/permute: stable by expert id
        ord.resize(A);
        for (size_t a = 0; a < A; ++a) ord[a] = int64_t(a);
        const int32_t* ids = idx[i];
        std::stable_sort(ord.begin(), ord.end(), [ids](int64_t x, int64_t y) { return ids[x] < ids[y]; });
    }
    return 0;
}

int oracle_moe_dispatch(int p, const void* const* x, const int32_t* const* idx, size_t T, int k, size_t H, int E,
                        int dtype, size_t cap_rows, void* const* recv, int64_t* expert_counts,
                        int32_t* const* pos, int64_t* recv_counts) {
    if (!valid_common(p, dtype)) return -1;
    MoeRoute R;
    if (moe_route(p, idx, T, k, E, &R) != 0) return -1;
    const size_t A = T * size_t(k), d = elem_size(dtype);
    // exchange counts + capacity: rows arriving at each destination
    std::vector<int64_t> rows_in(p, 0);
    for (int i = 0; i < p; ++i)
        for (int j = 0; j < p; ++j) rows_in[j] += R.c[size_t(i) * p + j];
    for (int j = 0; j < p; ++j)
        if (size_t(rows_in[j]) > cap_rows) return 1;
    // pack: send_i holds rank i's rows in packed order
    std::vector<std::vector<unsigned char>> send(p);
    std::vector<const void*> send_ptrs(p);
    for (int i = 0; i < p; ++i) {
        send[i].resize(std::max<size_t>(A * H * d, 1));
        for (size_t q = 0; q < A; ++q) {
            const size_t t = size_t(R.order[i][q]) / size_t(k);
            std::memcpy(send[i].data() + q * H * d, static_cast<const char*>(x[i]) + t * H * d, H * d);
        }
        send_ptrs[i] = send[i].data();
    }
    // variable-split exchange: element counts are rows times H
    std::vector<int64_t> ce(size_t(p) * p);
    for (size_t a = 0; a < ce.size(); ++a) ce[a] = R.c[a] * int64_t(H);
    if (oracle_alltoallv(p, send_ptrs.data(), recv, ce.data(), dtype, nullptr) != 0) return -1;
    // where every assignment landed: its row in the owner's receive buffer
    if (pos) {
        for (int i = 0; i < p; ++i) {
            for (size_t q = 0; q < A; ++q) {
                const int64_t a = R.order[i][q];
                const int j = idx[i][a] / R.E_loc;
                int64_t sdispl = 0, rdispl = 0;
                for (int jj = 0; jj < j; ++jj) sdispl += R.c[size_t(i) * p + jj];
                for (int ii = 0; ii < i; ++ii) rdispl += R.c[size_t(ii) * p + j];
                pos[i][a] = int32_t(rdispl + (int64_t(q) - sdispl));
            }
        }
    }
    if (expert_counts)
        for (int i = 0; i < p; ++i)
            for (int e = 0; e < E; ++e) expert_counts[size_t(i) * E + e] = R.cnt[i][e];
    if (recv_counts)
        for (int j = 0; j < p; ++j) recv_counts[j] = rows_in[j];
    return 0;
}

int oracle_moe_combine(int p, const void* const* y, const int32_t* const* idx, const float* const* w,
                       const void* const* residual, size_t T, int k, size_t H, int E, int dtype, void* const* out,
                       int acc) {
    if (p < 1 || (dtype != DT_FP32 && dtype != DT_BF16) || (acc != ACC_EXACT && acc != ACC_RANKFOLD)) return -1;
    MoeRoute R;
    if (moe_route(p, idx, T, k, E, &R) != 0) return -1;
    const size_t A = T * size_t(k), d = elem_size(dtype);
    // reverse variable-split exchange (counts transposed): back_i holds, in packed order, the rows
    // the experts returned for rank i's assignments
    std::vector<std::vector<unsigned char>> back(p);
    std::vector<void*> back_ptrs(p);
    for (int i = 0; i < p; ++i) {
        back[i].assign(std::max<size_t>(A * H * d, 1), 0);
        back_ptrs[i] = back[i].data();
    }
    std::vector<int64_t> ct(size_t(p) * p);
    for (int i = 0; i < p; ++i)
        for (int j = 0; j < p; ++j) ct[size_t(j) * p + i] = R.c[size_t(i) * p + j] * int64_t(H);
    if (oracle_alltoallv(p, y, back_ptrs.data(), ct.data(), dtype, nullptr) != 0) return -1;
    // unpermute + weighted combine
    for (int i = 0; i < p; ++i) {
        std::vector<int64_t> qpos(A);
        for (size_t q = 0; q < A; ++q) qpos[size_t(R.order[i][q])] = int64_t(q);
        for (size_t t = 0; t < T; ++t) {
            for (size_t h = 0; h < H; ++h) {
                if (acc == ACC_EXACT) {
                    double sum = residual ? load_as_double(residual[i], dtype, t * H + h) : 0.0;
                    for (int s = 0; s < k; ++s) {
                        const size_t q = size_t(qpos[t * k + s]);
                        sum += double(w[i][t * k + s]) * load_as_double(back[i].data(), dtype, q * H + h);
                    }
                    store_double_rounded_once(out[i], dtype, t * H + h, sum);
                } else {
                    float f;
                    int s0 = 0;
                    if (residual) {
                        f = load_as_float(residual[i], dtype, t * H + h);
                    } else {
                        f = w[i][t * k] * load_as_float(back[i].data(), dtype, size_t(qpos[t * k]) * H + h);
                        s0 = 1;
                    }
                    for (int s = s0; s < k; ++s) {
                        const size_t q = size_t(qpos[t * k + s]);
                        f = f + w[i][t * k + s] * load_as_float(back[i].data(), dtype, q * H + h);
                    }
                    store_float(out[i], dtype, t * H + h, f);
                }
            }
        }
    }
    return 0;
}

/* ===================== helpers the tests pin directly ============================================ */

uint16_t oracle_float_to_bf16(float f) { return float_to_bf16_rne(f); }
uint16_t oracle_double_to_bf16(double x) { return double_to_bf16_rne(x); }
float oracle_bf16_to_float(uint16_t h) { return bf16_to_float(h); }

/* The ring segment rule, exposed so a test can pin it against the page's even split. */
void oracle_ring_segment(size_t n, int p, int k, size_t* begin, size_t* end) { ring_segment(n, p, k, begin, end); }

}  // extern "C"
