// vmm.cu -- per-rank [E+B, H, H'] weight views built with CUDA virtual memory.
//
// The pages describe one contiguous symmetric-memory weight tensor per expert
// projection, [E+B, H, H'], whose rows the grouped GEMM addresses by index
// ("Moonshot AI Open-Sources MoonEP ..." on ainovat.com, the contract
// paragraph).  With R logical ranks on one GPU the same picture is built
// from address-space aliasing: one physical block holds the E home experts and
// is mapped at the start of every rank's view, and each rank maps its own
// physical block of B slots behind it.  Every view is contiguous, a home
// expert exists once in memory, and a slot write is private to its rank.
// The R views are reserved as one address range, view r at r * view_bytes,
// so that a consumer can address all of them from one base pointer (the
// grouped expert GEMM builds a single TMA tensor map over them).
//
// The driver's virtual-memory calls are taken through cudaGetDriverEntryPoint
// so that the library does not link against the driver library itself.
#include <cuda.h>

#include <cstring>
#include <new>

#include "internal.cuh"

namespace moonep {
namespace {

using PFN_GetGran = CUresult (*)(size_t*, const CUmemAllocationProp*,
                                 CUmemAllocationGranularity_flags);
using PFN_Create = CUresult (*)(CUmemGenericAllocationHandle*, size_t, const CUmemAllocationProp*,
                                unsigned long long);
using PFN_Release = CUresult (*)(CUmemGenericAllocationHandle);
using PFN_Reserve = CUresult (*)(CUdeviceptr*, size_t, size_t, CUdeviceptr, unsigned long long);
using PFN_Free = CUresult (*)(CUdeviceptr, size_t);
using PFN_Map = CUresult (*)(CUdeviceptr, size_t, size_t, CUmemGenericAllocationHandle,
                             unsigned long long);
using PFN_Unmap = CUresult (*)(CUdeviceptr, size_t);
using PFN_SetAccess = CUresult (*)(CUdeviceptr, size_t, const CUmemAccessDesc*, size_t);

struct Driver {
    PFN_GetGran gran = nullptr;
    PFN_Create create = nullptr;
    PFN_Release release = nullptr;
    PFN_Reserve reserve = nullptr;
    PFN_Free free_va = nullptr;
    PFN_Map map = nullptr;
    PFN_Unmap unmap = nullptr;
    PFN_SetAccess access = nullptr;
    bool ok = false;
};

template <typename F>
bool entry(const char* name, F* out) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return false;
    *out = reinterpret_cast<F>(fn);
    return true;
}

const Driver& driver() {
    static Driver d = [] {
        Driver x;
        x.ok = entry("cuMemGetAllocationGranularity", &x.gran) && entry("cuMemCreate", &x.create) &&
               entry("cuMemRelease", &x.release) && entry("cuMemAddressReserve", &x.reserve) &&
               entry("cuMemAddressFree", &x.free_va) && entry("cuMemMap", &x.map) &&
               entry("cuMemUnmap", &x.unmap) && entry("cuMemSetAccess", &x.access);
        return x;
    }();
    return d;
}

struct Impl {
    int R = 0;
    size_t home_bytes = 0, slot_bytes = 0, view_bytes = 0;
    CUmemGenericAllocationHandle home = 0;
    bool home_made = false;
    CUmemGenericAllocationHandle slot[MOONEP_MAX_R] = {};
    bool slot_made[MOONEP_MAX_R] = {};
    CUdeviceptr base = 0;  // one reservation of R * view_bytes
    CUdeviceptr va[MOONEP_MAX_R] = {};
    bool home_mapped[MOONEP_MAX_R] = {};
    bool slot_mapped[MOONEP_MAX_R] = {};
};

void teardown(Impl* m) {
    const Driver& d = driver();
    for (int r = 0; r < m->R; ++r) {
        if (m->slot_mapped[r]) d.unmap(m->va[r] + m->home_bytes, m->slot_bytes);
        if (m->home_mapped[r]) d.unmap(m->va[r], m->home_bytes);
        if (m->slot_made[r]) d.release(m->slot[r]);
    }
    if (m->base) d.free_va(m->base, m->view_bytes * m->R);
    if (m->home_made) d.release(m->home);
}

}  // namespace

int weights_create(const moonep_config& c, int elem_bytes, moonep_weights_t* out,
                   const char** why) {
    const Driver& d = driver();
    if (!d.ok) {
        *why = "CUDA virtual-memory entry points are unavailable";
        return MOONEP_ERR_CUDA;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        *why = "no current CUDA device";
        return MOONEP_ERR_CUDA;
    }
    CUmemAllocationProp prop;
    std::memset(&prop, 0, sizeof(prop));
    prop.type = CU_MEM_ALLOCATION_TYPE_PINNED;
    prop.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
    prop.location.id = dev;
    size_t gran = 0;
    if (d.gran(&gran, &prop, CU_MEM_ALLOC_GRANULARITY_MINIMUM) != CUDA_SUCCESS || gran == 0) {
        *why = "cuMemGetAllocationGranularity failed";
        return MOONEP_ERR_CUDA;
    }
    const size_t row = (size_t)c.H * c.Hp * elem_bytes;
    if (row % gran != 0) {
        *why = "H*Hp*elem_bytes is not a multiple of the allocation granularity";
        return MOONEP_ERR_INVALID_ARG;
    }
    Impl* m = new (std::nothrow) Impl();
    if (!m) {
        *why = "out of host memory";
        return MOONEP_ERR_CUDA;
    }
    m->R = c.R;
    m->home_bytes = row * c.E;
    m->slot_bytes = row * c.B;
    m->view_bytes = m->home_bytes + m->slot_bytes;
    CUmemAccessDesc acc;
    std::memset(&acc, 0, sizeof(acc));
    acc.location = prop.location;
    acc.flags = CU_MEM_ACCESS_FLAGS_PROT_READWRITE;

    bool fail = d.create(&m->home, m->home_bytes, &prop, 0) != CUDA_SUCCESS;
    m->home_made = !fail;
    if (!fail) {
        fail = d.reserve(&m->base, m->view_bytes * c.R, gran, 0, 0) != CUDA_SUCCESS;
        if (fail) m->base = 0;
    }
    for (int r = 0; r < c.R && !fail; ++r) {
        if (c.B > 0) {
            fail = d.create(&m->slot[r], m->slot_bytes, &prop, 0) != CUDA_SUCCESS;
            m->slot_made[r] = !fail;
            if (fail) break;
        }
        m->va[r] = m->base + (CUdeviceptr)r * m->view_bytes;
        fail = d.map(m->va[r], m->home_bytes, 0, m->home, 0) != CUDA_SUCCESS;
        m->home_mapped[r] = !fail;
        if (fail) break;
        if (c.B > 0) {
            fail = d.map(m->va[r] + m->home_bytes, m->slot_bytes, 0, m->slot[r], 0) != CUDA_SUCCESS;
            m->slot_mapped[r] = !fail;
            if (fail) break;
        }
        fail = d.access(m->va[r], m->view_bytes, &acc, 1) != CUDA_SUCCESS;
    }
    if (fail) {
        teardown(m);
        delete m;
        *why = "CUDA virtual-memory allocation or mapping failed (out of memory?)";
        return MOONEP_ERR_CUDA;
    }
    std::memset(out, 0, sizeof(*out));
    for (int r = 0; r < c.R; ++r) out->rank_view[r] = reinterpret_cast<void*>(m->va[r]);
    out->row_bytes = row;
    out->view_bytes = m->view_bytes;
    out->R = c.R;
    out->E = c.E;
    out->B = c.B;
    out->elem_bytes = elem_bytes;
    out->impl = m;
    return MOONEP_OK;
}

int weights_destroy(moonep_weights_t* w) {
    if (!w || !w->impl) return MOONEP_ERR_INVALID_ARG;
    Impl* m = static_cast<Impl*>(w->impl);
    cudaDeviceSynchronize();
    teardown(m);
    delete m;
    w->impl = nullptr;
    return MOONEP_OK;
}

}  // namespace moonep
