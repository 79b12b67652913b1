// Run-time loading of the NCCL entry points (see nccl_dl.h).
#include "nccl_dl.h"

#include <dlfcn.h>

#include <mutex>

namespace mt {

namespace {

template <typename F>
bool resolve(void* h, const char* name, F* out) {
  *out = reinterpret_cast<F>(dlsym(h, name));
  return *out != nullptr;
}

}  // namespace

const NcclApi* nccl_api(std::string* why) {
  static NcclApi api;
  static std::string error;
  static std::once_flag once;
  std::call_once(once, [] {
    void* h = dlopen("libnccl.so.2", RTLD_NOW | RTLD_GLOBAL);
    if (!h) {
      const char* e = dlerror();
      error = std::string("cannot load libnccl.so.2: ") + (e ? e : "unknown error");
      return;
    }
    NcclApi a;
    const bool ok = resolve(h, "ncclGetUniqueId", &a.GetUniqueId) && resolve(h, "ncclCommInitRank", &a.CommInitRank) &&
                    resolve(h, "ncclCommSplit", &a.CommSplit) && resolve(h, "ncclCommDestroy", &a.CommDestroy) &&
                    resolve(h, "ncclAllGather", &a.AllGather) && resolve(h, "ncclReduceScatter", &a.ReduceScatter) &&
                    resolve(h, "ncclAllReduce", &a.AllReduce) && resolve(h, "ncclGetErrorString", &a.GetErrorString);
    if (!ok) {
      error = "libnccl.so.2 lacks an entry point this library needs (NCCL 2.18 or later)";
      return;
    }
    api = a;
  });
  if (!api.GetUniqueId) {
    if (why) *why = error;
    return nullptr;
  }
  return &api;
}

}  // namespace mt
