// arena.cuh - dllm_arena: one fixed device virtual address range whose prefix is backed by
// physical memory on demand (the global memory manager with virtual memory mapping of the
// Mosaic page, TL;DR and Abstract; Fig. 4 compares the memory it reserves with the
// theoretical peak).
//
// The range is reserved once with cuMemAddressReserve and never moves.  Physical memory is
// created (cuMemCreate), mapped (cuMemMap) and made read-write for the owning device
// (cuMemSetAccess) in fixed chunks: chunk i always backs [i * chunk, (i + 1) * chunk), so
// growing maps chunks past the current end and shrinking unmaps and releases chunks from
// the end.  A decode step's workspace grows with its masked count
// (dllm_workspace_bytes_rows); mapping just that much keeps the device memory held close
// to the step's own requirement instead of the worst case over every mask.
//
// Host code only.  The driver's virtual-memory calls are resolved at run time through the
// runtime's driver entry-point query, as the tensor-map encoder is, so the library does not
// link libcuda directly.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "dllm.h"

struct dllm_arena {
  int device = 0;
  CUdeviceptr base = 0;
  size_t reserved = 0;
  size_t chunk = 0;
  std::vector<CUmemGenericAllocationHandle> handles;   // handles[i] backs chunk i
};

namespace dllm {
namespace arena {

struct Driver {
  bool ok = false;
  CUresult (*granularity)(size_t*, const CUmemAllocationProp*, CUmemAllocationGranularity_flags) = nullptr;
  CUresult (*reserve)(CUdeviceptr*, size_t, size_t, CUdeviceptr, unsigned long long) = nullptr;
  CUresult (*free_va)(CUdeviceptr, size_t) = nullptr;
  CUresult (*create)(CUmemGenericAllocationHandle*, size_t, const CUmemAllocationProp*,
                     unsigned long long) = nullptr;
  CUresult (*release)(CUmemGenericAllocationHandle) = nullptr;
  CUresult (*map)(CUdeviceptr, size_t, size_t, CUmemGenericAllocationHandle, unsigned long long) = nullptr;
  CUresult (*unmap)(CUdeviceptr, size_t) = nullptr;
  CUresult (*set_access)(CUdeviceptr, size_t, const CUmemAccessDesc*, size_t) = nullptr;
};

template <class F>
bool resolve(const char* name, F* fn) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || p == nullptr)
    return false;
  *fn = reinterpret_cast<F>(p);
  return true;
}

inline const Driver& driver() {
  static Driver d;
  static std::once_flag once;
  std::call_once(once, [] {
    d.ok = resolve("cuMemGetAllocationGranularity", &d.granularity) &&
           resolve("cuMemAddressReserve", &d.reserve) && resolve("cuMemAddressFree", &d.free_va) &&
           resolve("cuMemCreate", &d.create) && resolve("cuMemRelease", &d.release) &&
           resolve("cuMemMap", &d.map) && resolve("cuMemUnmap", &d.unmap) &&
           resolve("cuMemSetAccess", &d.set_access);
  });
  return d;
}

inline CUmemAllocationProp device_prop(int dev) {
  CUmemAllocationProp prop = {};
  prop.type = CU_MEM_ALLOCATION_TYPE_PINNED;
  prop.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
  prop.location.id = dev;
  return prop;
}

// Unmap and release chunks from the end until `keep` remain.
inline bool trim(dllm_arena* a, size_t keep) {
  const Driver& d = driver();
  bool ok = true;
  while (a->handles.size() > keep) {
    const size_t i = a->handles.size() - 1;
    if (d.unmap(a->base + i * a->chunk, a->chunk) != CUDA_SUCCESS) ok = false;
    if (d.release(a->handles[i]) != CUDA_SUCCESS) ok = false;
    a->handles.pop_back();
  }
  return ok;
}

}  // namespace arena
}  // namespace dllm

extern "C" {

dllm_status dllm_arena_create(size_t reserve_bytes, size_t chunk_bytes, dllm_arena** out) {
  using namespace dllm::arena;
  if (out == nullptr) return DLLM_ERR_NULL;
  *out = nullptr;
  if (reserve_bytes == 0) return DLLM_ERR_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DLLM_ERR_CUDA;
  cudaDeviceProp p;
  if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return DLLM_ERR_CUDA;
  if (p.major != 10 || p.minor != 0) return DLLM_ERR_DEVICE;
  if (cudaFree(nullptr) != cudaSuccess) return DLLM_ERR_CUDA;     // the device's context exists
  const Driver& d = driver();
  if (!d.ok) return DLLM_ERR_CUDA;
  const CUmemAllocationProp prop = device_prop(dev);
  size_t gran = 0;
  if (d.granularity(&gran, &prop, CU_MEM_ALLOC_GRANULARITY_MINIMUM) != CUDA_SUCCESS || gran == 0)
    return DLLM_ERR_CUDA;
  const size_t chunk = chunk_bytes == 0 ? gran : (chunk_bytes + gran - 1) / gran * gran;
  const size_t reserved = (reserve_bytes + chunk - 1) / chunk * chunk;
  CUdeviceptr base = 0;
  if (d.reserve(&base, reserved, gran, 0, 0) != CUDA_SUCCESS) return DLLM_ERR_CUDA;
  dllm_arena* a = new dllm_arena;
  a->device = dev;
  a->base = base;
  a->reserved = reserved;
  a->chunk = chunk;
  *out = a;
  return DLLM_OK;
}

dllm_status dllm_arena_map(dllm_arena* a, size_t bytes) {
  using namespace dllm::arena;
  if (a == nullptr) return DLLM_ERR_NULL;
  if (bytes > a->reserved) return DLLM_ERR_SHAPE;
  const Driver& d = driver();
  const size_t want = (bytes + a->chunk - 1) / a->chunk;
  const size_t have = a->handles.size();
  if (want > have) {
    const CUmemAllocationProp prop = device_prop(a->device);
    CUmemAccessDesc acc = {};
    acc.location.type = CU_MEM_LOCATION_TYPE_DEVICE;
    acc.location.id = a->device;
    acc.flags = CU_MEM_ACCESS_FLAGS_PROT_READWRITE;
    for (size_t i = have; i < want; ++i) {
      CUmemGenericAllocationHandle h;
      if (d.create(&h, a->chunk, &prop, 0) != CUDA_SUCCESS) {
        trim(a, have);
        return DLLM_ERR_CUDA;
      }
      const CUdeviceptr at = a->base + i * a->chunk;
      if (d.map(at, a->chunk, 0, h, 0) != CUDA_SUCCESS) {
        d.release(h);
        trim(a, have);
        return DLLM_ERR_CUDA;
      }
      a->handles.push_back(h);
      // access per chunk: a chunk unmapped later is then referenced by nothing else (an
      // access range spanning several chunks kept released chunks allocated)
      if (d.set_access(at, a->chunk, &acc, 1) != CUDA_SUCCESS) {
        trim(a, have);
        return DLLM_ERR_CUDA;
      }
    }
  } else if (want < have) {
    // no kernel still running may touch a chunk that is about to be released
    if (cudaDeviceSynchronize() != cudaSuccess) return DLLM_ERR_CUDA;
    if (!trim(a, want)) return DLLM_ERR_CUDA;
  }
  return DLLM_OK;
}

void* dllm_arena_ptr(const dllm_arena* a) {
  return a == nullptr ? nullptr : reinterpret_cast<void*>(static_cast<uintptr_t>(a->base));
}

size_t dllm_arena_reserved(const dllm_arena* a) { return a == nullptr ? 0 : a->reserved; }

size_t dllm_arena_mapped(const dllm_arena* a) {
  return a == nullptr ? 0 : a->handles.size() * a->chunk;
}

size_t dllm_arena_chunk(const dllm_arena* a) { return a == nullptr ? 0 : a->chunk; }

dllm_status dllm_arena_destroy(dllm_arena* a) {
  using namespace dllm::arena;
  if (a == nullptr) return DLLM_OK;
  dllm_status st = DLLM_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) st = DLLM_ERR_CUDA;
  if (!trim(a, 0)) st = DLLM_ERR_CUDA;
  if (driver().free_va(a->base, a->reserved) != CUDA_SUCCESS) st = DLLM_ERR_CUDA;
  delete a;
  return st;
}

}  // extern "C"
