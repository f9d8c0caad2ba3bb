// The shared-prefix plan of the decode step (nvpa_decode_step_shared_prefix).
#include <mutex>

#include "decode_params.cuh"

namespace nvpa {

// ------------------------------------------------------------------------------------
// shared-prefix plan
// ------------------------------------------------------------------------------------
// Prefix caching hands a cached prompt's blocks to every sequence that starts with it, by
// reference count ("Nano-vLLM part 1" section 4.2), so such sequences' block tables begin
// with the same physical block ids.  This plan buckets the sequences by their first block
// id (open addressing in shared memory); a bucket with at least min_members sequences is a
// group, and the group's prefix is the longest run of leading blocks that every member
// holds, counting only blocks that lie wholly before each member's newest token (that
// token is written in this step).  Each member's context then splits into
//   prefix partitions  0 .. npc-1       keys [c * pchunk, ...) of the prefix, computed once
//                                        for all members on the tensor cores;
//   private partitions npc .. npc+nsp-1 keys [prefix + s * chunk, ...), worker items;
// and the combine merges all npc + nsp partials.  Sequences outside a group get the plain
// decode plan's items.  Counters in the workspace: [0] items claimed after the worker's
// first round, [1] items, [2] groups, [3] members, [4] prefix work units (pairs of query
// tiles of one group and partition), [5] the prefix kernel's unit counter.

__global__ void __launch_bounds__(1024) decode_plan_shared_kernel(const AttnParams p) {
    extern __shared__ int sh[];
    int* tkey = sh;                            // first block id of the bucket, -1 = empty
    int* tlead = tkey + kSharedTable;          // smallest member; later the member fill count
    int* tcnt = tlead + kSharedTable;          // sequences in the bucket
    int* tpref = tcnt + kSharedTable;          // prefix blocks: min over the members
    int* tgid = tpref + kSharedTable;          // group id, -1 = not a group
    int* tmst = tgid + kSharedTable;           // first index of the group in members[]
    int* s_slot = tmst + kSharedTable;         // bucket of each sequence; later its prefix tokens
    int* s_ctx = s_slot + kSharedMaxBatch;     // clamped context length
    __shared__ int warp_tot[32];
    __shared__ int s_ntiles;
    const int tid = threadIdx.x;
    pdl_launch_dependents();
    for (int i = tid; i < kSharedTable; i += blockDim.x) {
        tkey[i] = -1;
        tlead[i] = INT_MAX;
        tcnt[i] = 0;
        tpref[i] = INT_MAX;
        tgid[i] = -1;
    }
    if (tid == 0) s_ntiles = 0;
    __syncthreads();
    const int lim = (int)min((long long)p.max_ctx, (long long)p.max_blocks * p.block_size);

    // 1. bucket by first block
    for (int b = tid; b < p.batch; b += blockDim.x) {
        int ctx = __ldg(p.context_lens + b);
        const int key = __ldg(p.block_tables + (size_t)b * p.max_blocks);   // loaded alongside
        if (ctx < 0 || ctx > lim) {
            flag_error(p.err, NVPA_FLAG_BAD_LENGTH);
            ctx = min(max(ctx, 0), lim);
        }
        s_ctx[b] = ctx;
        int slot = -1;
        const int full = ctx > 0 ? (ctx - 1) >> p.block_shift : 0;   // blocks before the newest token
        if (full >= 1) {
            if (key >= 0 && key < p.num_blocks) {
                int h = (int)(((uint32_t)key * 2654435761u) >> 20) & (kSharedTable - 1);
                while (true) {   // at most batch < kSharedTable buckets are taken
                    const int prev = atomicCAS(tkey + h, -1, key);
                    if (prev == -1 || prev == key) break;
                    h = (h + 1) & (kSharedTable - 1);
                }
                slot = h;
                atomicMin(tlead + h, b);
                atomicAdd(tcnt + h, 1);
            }
        }
        s_slot[b] = slot;
    }
    __syncthreads();

    // 2. prefix of each bucket that is large enough: common leading blocks with its
    //    smallest member, at most the blocks before each member's newest token
    for (int b = tid; b < p.batch; b += blockDim.x) {
        const int slot = s_slot[b];
        if (slot < 0 || tcnt[slot] < p.min_members) continue;
        const int full = (s_ctx[b] - 1) >> p.block_shift;
        const int32_t* bb = p.block_tables + (size_t)b * p.max_blocks;
        const int32_t* bl = p.block_tables + (size_t)tlead[slot] * p.max_blocks;
        // common leading blocks with the smallest member, compared 8 entries at a time
        // (independent loads); block 0 is the bucket key
        int n = 1;
        bool run = true;
        while (run && n < full) {
            int eb[8], el[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool in = n + u < full;
                eb[u] = in ? __ldg(bb + n + u) : 0;
                el[u] = in ? __ldg(bl + n + u) : 1;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (run && eb[u] == el[u]) ++n;
                else run = false;
            }
        }
        atomicMin(tpref + slot, n);
    }
    __syncthreads();

    // 3. number the groups (in bucket order), place their member lists, list their tiles
    constexpr int PER = kSharedTable / 1024;
    bool used[PER];
    int v = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int i = tid * PER + u;
        used[u] = i < kSharedTable && tkey[i] >= 0 && tcnt[i] >= p.min_members && tpref[i] != INT_MAX;
        if (used[u]) v += (tcnt[i] << 12) + 1;   // members in the high bits, groups in the low 12
    }
    int tot = 0;
    int excl = block_exclusive_scan(v, warp_tot, tot);
    int g = excl & 4095, m = excl >> 12;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        if (!used[u]) continue;
        const int i = tid * PER + u;
        const int cnt = tcnt[i];
        const int pre = tpref[i] << p.block_shift;
        tgid[i] = g;
        tmst[i] = m;
        tlead[i] = 0;
        p.group_start[g] = m;
        p.group_len[g] = pre;
        // query tiles of the group in pairs (the tensor-core kernel's work unit), for
        // every prefix partition
        const int nq = (cnt + p.ptq - 1) / p.ptq;
        const int npair = (nq + 1) / 2;
        const int nch = (pre + p.pchunk - 1) / p.pchunk;
        const int off = atomicAdd(&s_ntiles, npair * nch);
        for (int c = 0; c < nch; ++c)
            for (int u = 0; u < npair; ++u)
                p.ptiles[off + c * npair + u] = make_int4(g, 2 * u, 2 * u + 1 < nq ? 2 * u + 1 : -1, c);
        ++g;
        m += cnt;
    }
    const int ngroups = tot & 4095, nmembers = tot >> 12;
    if (tid == 0) p.group_start[ngroups] = nmembers;
    __syncthreads();

    // 4. members and partition counts
    for (int b = tid; b < p.batch; b += blockDim.x) {
        const int slot = s_slot[b];
        const int gid = slot >= 0 ? tgid[slot] : -1;
        int pre = 0;
        if (gid >= 0) {
            const int pos = atomicAdd(tlead + slot, 1);
            p.members[tmst[slot] + pos] = b;
            pre = tpref[slot] << p.block_shift;
        }
        const int npc = (pre + p.pchunk - 1) / p.pchunk;
        const int nsp = max(1, (s_ctx[b] - pre + p.chunk - 1) / p.chunk);
        p.nsplit[b] = npc + nsp;
        s_slot[b] = pre;
    }
    __syncthreads();

    // 5. worker items for the private partitions
    // Every full-length partition first, sequence by sequence, then each sequence's last,
    // shorter partition, longest first (a counting sort over 256 length classes): the
    // items claimed last are the shortest, so the worker's warps finish close together.
    __shared__ int s_cls[kLengthClasses];
    for (int i = tid; i < kLengthClasses; i += blockDim.x) s_cls[i] = 0;
    __syncthreads();
    int carry = 0;
    for (int base = 0; base < p.batch; base += blockDim.x) {
        const int b = base + tid;
        int nfull = 0, npc = 0, nsp = 0, pre = 0;
        if (b < p.batch) {
            pre = s_slot[b];
            const int priv = s_ctx[b] - pre;
            npc = (pre + p.pchunk - 1) / p.pchunk;
            nsp = max(1, (priv + p.chunk - 1) / p.chunk);
            const int last = priv - (nsp - 1) * p.chunk;
            nfull = last == p.chunk ? nsp : nsp - 1;
            if (last < p.chunk) atomicAdd(s_cls + length_class(last, p.chunk), 1);
        }
        int block_tot = 0;
        const int e = carry + block_exclusive_scan(nfull, warp_tot, block_tot);
        for (int s = 0; s < nfull; ++s)
            p.items[e + s] = make_int4(b, (npc + s) | ((npc + nsp) << 16), pre + s * p.chunk, pre + (s + 1) * p.chunk);
        carry += block_tot;
    }
    __syncthreads();
    // first position of each length class, longest class first, after the full partitions
    {
        const int cls = kLengthClasses - 1 - tid;
        const int v = tid < kLengthClasses ? s_cls[cls] : 0;
        int tot_short = 0;
        const int e = block_exclusive_scan(v, warp_tot, tot_short);
        if (tid < kLengthClasses) s_cls[cls] = carry + e;
        __syncthreads();
        for (int b = tid; b < p.batch; b += blockDim.x) {
            const int pre = s_slot[b], ctx = s_ctx[b];
            const int priv = ctx - pre;
            const int npc = (pre + p.pchunk - 1) / p.pchunk;
            const int nsp = max(1, (priv + p.chunk - 1) / p.chunk);
            const int last = priv - (nsp - 1) * p.chunk;
            if (last == p.chunk) continue;
            const int pos = atomicAdd(s_cls + length_class(last, p.chunk), 1);
            p.items[pos] = make_int4(b, (npc + nsp - 1) | ((npc + nsp) << 16), pre + (nsp - 1) * p.chunk, ctx);
        }
        carry += tot_short;
    }
    if (tid == 0) {
        p.counter[0] = 0;
        p.counter[1] = carry * p.hkv;
        p.counter[2] = ngroups;
        p.counter[3] = nmembers;
        p.counter[4] = s_ntiles;
        p.counter[5] = 0;   // the prefix kernel's unit counter
    }
}


cudaError_t launch_decode_plan_shared(const AttnParams& p, cudaStream_t stream) {
    static std::once_flag once[64];
    int dev = 0;
    cudaGetDevice(&dev);
    std::call_once(once[dev & 63], [] {
        cudaFuncSetAttribute(decode_plan_shared_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSharedPlanSmem);
    });
    decode_plan_shared_kernel<<<1, 1024, kSharedPlanSmem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace nvpa
