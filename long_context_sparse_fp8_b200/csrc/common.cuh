// common.cuh -- shared device helpers of libdsa (views of the ABI structs, batch
// row lookup, element loads and the device check word).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

enum DType : int { kF32 = 0, kBF16 = 1, kE4M3 = 2 };

enum CheckCode : int { kCheckNone = 0, kCheckBadPage = 1, kCheckBadIndex = 2, kCheckBadBatch = 3,
                       kCheckTimeout = 4, kCheckFp16Range = 5 };

// Plain copies of the ABI structs passed to kernels by value.
struct BatchView {
    int num_seqs;
    int total_q;
    int max_seq_len;
    const int* cu_q;      // [B+1]
    const int* seq_lens;  // [B]
};

struct CacheView {
    const void* data;     // [num_pages][page_size][dim]
    const float* scale;   // [num_pages][page_size] or nullptr
    const int* table;     // [B][bt_stride]
    long long num_pages;
    int page_size;
    int dim;
    int bt_stride;
    int dtype;
};

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while its predecessor in the stream still runs: it must
// execute pdl_wait() before touching anything the predecessor writes (returns at
// once when there is no such predecessor).  pdl_trigger() lets the successor be
// scheduled before this grid ends.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ void report(int* check, int code) {
    if (check) atomicCAS(check, 0, code);
}

// Largest b in [0, B) with cu_q[b] <= t: the sequence that owns query row t
// (empty sequences share their cu_q value with the next one and are skipped).
__device__ __forceinline__ int find_seq(const int* __restrict__ cu_q, int num_seqs, int t) {
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu_q + mid) <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

struct RowInfo {
    int b;     // sequence
    int pos;   // position of the query token; keys 0..pos are visible
    bool ok;
};

// Query row t is token L_b - nq_b + (t - cu_q[b]) of its sequence.
__device__ __forceinline__ RowInfo row_info(const BatchView& bv, int t, int* check) {
    RowInfo r;
    r.b = find_seq(bv.cu_q, bv.num_seqs, t);
    int q0 = __ldg(bv.cu_q + r.b), q1 = __ldg(bv.cu_q + r.b + 1);
    int L = __ldg(bv.seq_lens + r.b);
    r.pos = L - (q1 - q0) + (t - q0);
    r.ok = (q1 - q0) <= L && L <= bv.max_seq_len && r.pos >= 0;
    if (!r.ok) report(check, kCheckBadBatch);
    return r;
}

// Physical row (page * page_size + offset) of logical token s of sequence b, or -1
// (and a recorded check) if the table entry is out of range.
__device__ __forceinline__ long long cache_row(const CacheView& c, int b, int s, int* check) {
    int page = __ldg(c.table + (long long)b * c.bt_stride + s / c.page_size);
    if (page < 0 || (long long)page >= c.num_pages) {
        report(check, kCheckBadPage);
        return -1;
    }
    return (long long)page * c.page_size + s % c.page_size;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
    __nv_fp8_e4m3 v;
    v.__x = b;
    return float(v);
}

template <int DT>
__device__ __forceinline__ float load_as_f32(const void* base, long long i) {
    if constexpr (DT == kF32) return __ldg(reinterpret_cast<const float*>(base) + i);
    else if constexpr (DT == kBF16)
        return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short*>(base) + i));
    else return e4m3_to_f32(__ldg(reinterpret_cast<const unsigned char*>(base) + i));
}

}  // namespace dsa
