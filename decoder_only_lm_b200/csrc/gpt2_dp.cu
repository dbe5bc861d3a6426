// Data-parallel gradient exchange inside the library [LECTURE: DDP, the
// gradients of the ranks averaged before the update, no exchange until the
// last micro-batch; CH28 §28.3: rank r reads the windows at B*T*r, advancing
// B*T*N].
//
// The handle owns an NCCL communicator over the N ranks of the job.  While it
// is set, every backward that exchanges (the default; see gpt2_dp_sync)
// enqueues, as soon as a gradient bucket is final (gpt2_grad_buckets: one
// bucket per layer's weight matrices, last layer first, then the embeddings
// and every vector), an all-reduce (average) of the bucket's ranges on a
// communication stream that first waits for the handle's stream at that
// point.  So the all-reduces of the later layers cross NVLink while the
// earlier layers' backward runs, and only the last bucket is exposed.  The
// handle's stream waits for the communication stream at the end of the
// backward.  Every call is stream-ordered, so the exchange is also recorded
// into the CUDA graph of gpt2_stream_begin (one optimizer step with the
// exchange inside).
//
// NCCL is opened at run time (dlopen of libnccl.so.2, the one the process
// already holds if PyTorch loaded it): nothing links against it, and a
// process that never calls gpt2_dp_init never touches it.

#include <dlfcn.h>
#include <nccl.h>

#include <mutex>
#include <string>

#include "dp_internal.h"
#include "kernels.h"

namespace {

struct NcclApi {
  ncclResult_t (*GetUniqueId)(ncclUniqueId*) = nullptr;
  ncclResult_t (*CommInitRank)(ncclComm_t*, int, ncclUniqueId, int) = nullptr;
  ncclResult_t (*AllReduce)(const void*, void*, size_t, ncclDataType_t, ncclRedOp_t, ncclComm_t,
                            cudaStream_t) = nullptr;
  ncclResult_t (*CommDestroy)(ncclComm_t) = nullptr;
  ncclResult_t (*GroupStart)() = nullptr;
  ncclResult_t (*GroupEnd)() = nullptr;
  const char* (*GetErrorString)(ncclResult_t) = nullptr;
  bool ok = false;
  std::string why;
};

const NcclApi& nccl() {
  static NcclApi api;
  static std::once_flag once;
  std::call_once(once, [] {
    void* lib = dlopen("libnccl.so.2", RTLD_NOW | RTLD_NOLOAD);
    if (!lib) lib = dlopen("libnccl.so.2", RTLD_NOW);
    if (!lib) {
      api.why = std::string("cannot open libnccl.so.2: ") + dlerror();
      return;
    }
    auto sym = [&](const char* n) { return dlsym(lib, n); };
    api.GetUniqueId = reinterpret_cast<decltype(api.GetUniqueId)>(sym("ncclGetUniqueId"));
    api.CommInitRank = reinterpret_cast<decltype(api.CommInitRank)>(sym("ncclCommInitRank"));
    api.AllReduce = reinterpret_cast<decltype(api.AllReduce)>(sym("ncclAllReduce"));
    api.CommDestroy = reinterpret_cast<decltype(api.CommDestroy)>(sym("ncclCommDestroy"));
    api.GroupStart = reinterpret_cast<decltype(api.GroupStart)>(sym("ncclGroupStart"));
    api.GroupEnd = reinterpret_cast<decltype(api.GroupEnd)>(sym("ncclGroupEnd"));
    api.GetErrorString = reinterpret_cast<decltype(api.GetErrorString)>(sym("ncclGetErrorString"));
    api.ok = api.GetUniqueId && api.CommInitRank && api.AllReduce && api.CommDestroy &&
             api.GroupStart && api.GroupEnd && api.GetErrorString;
    if (!api.ok) api.why = "libnccl.so.2 lacks an entry point";
  });
  return api;
}

}  // namespace

namespace gpt2_internal {

int dp_allreduce_ranges(void* comm, const std::vector<std::pair<int64_t, int64_t>>& ranges,
                        float* grad, cudaStream_t st) {
  const NcclApi& n = nccl();
  ncclComm_t c = static_cast<ncclComm_t>(comm);
  ncclResult_t r = n.GroupStart();
  for (size_t k = 0; r == ncclSuccess && k < ranges.size(); ++k) {
    float* p = grad + ranges[k].first;
    r = n.AllReduce(p, p, size_t(ranges[k].second), ncclFloat32, ncclAvg, c, st);
  }
  const ncclResult_t r2 = n.GroupEnd();
  if (r == ncclSuccess) r = r2;
  if (r != ncclSuccess) {
    set_error(std::string("gradient all-reduce: ") + n.GetErrorString(r));
    return GPT2_ERR_CUDA;
  }
  return GPT2_OK;
}

int dp_comm_init(void** comm, const char* id, int rank, int world) {
  const NcclApi& n = nccl();
  if (!n.ok) {
    set_error("data parallel: " + n.why);
    return GPT2_ERR_CUDA;
  }
  ncclUniqueId uid;
  static_assert(sizeof(uid.internal) == GPT2_DP_ID_BYTES, "unique id size");
  memcpy(uid.internal, id, GPT2_DP_ID_BYTES);
  ncclComm_t c = nullptr;
  const ncclResult_t r = n.CommInitRank(&c, world, uid, rank);
  if (r != ncclSuccess) {
    set_error(std::string("ncclCommInitRank: ") + n.GetErrorString(r));
    return GPT2_ERR_CUDA;
  }
  *comm = c;
  return GPT2_OK;
}

void dp_comm_destroy(void* comm) {
  if (comm && nccl().ok) nccl().CommDestroy(static_cast<ncclComm_t>(comm));
}

}  // namespace gpt2_internal

extern "C" int gpt2_dp_unique_id(char* id) {
  if (!id) return GPT2_ERR_ARG;
  const NcclApi& n = nccl();
  if (!n.ok) {
    gpt2_internal::set_error("data parallel: " + n.why);
    return GPT2_ERR_CUDA;
  }
  ncclUniqueId uid;
  const ncclResult_t r = n.GetUniqueId(&uid);
  if (r != ncclSuccess) {
    gpt2_internal::set_error(std::string("ncclGetUniqueId: ") + n.GetErrorString(r));
    return GPT2_ERR_CUDA;
  }
  memcpy(id, uid.internal, GPT2_DP_ID_BYTES);
  return GPT2_OK;
}
