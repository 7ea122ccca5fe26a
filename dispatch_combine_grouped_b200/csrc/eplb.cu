// Redundant expert slots (EPLB): plan, replica assignment, weight placement; and the
// capacity cut, which needs the same per-expert rank of each assignment.
//
// "Wide EP：当 MoE Expert Parallel 横跨几十张 GPU", sections "为什么要把 EP 做宽"
// (E logical experts + R copies = E + R physical experts, E_local = (E + R) / P_e per
// owner), "Expert 副本在 Wide EP 中还有整除作用" (copies of hot experts, slot counts that
// divide the EP width, a logical expert's assignments spread over its copies) and
// "三种负载必须同时平衡" (the balancer minimises the largest expert / receive load).  The
// router's choice is kept: only which copy of the chosen expert serves an assignment
// changes ("Group-limited routing").
//
// The pages give the goal, not an algorithm; this file implements these steps:
//   plan   1. copies: each expert keeps one; each of the R extra copies in turn goes to
//             the expert with the largest load per copy, load_e / r_e (ties: lower id).
//          2. copy c of expert e carries floor(load_e / r_e) + (c < load_e mod r_e), the
//             rows step 4 gives it.  Copies are placed in descending load order (ties:
//             lower expert, lower copy) on the owner with free room that holds no copy
//             of the same expert if there is one, then the least loaded, then the lower.
//          3. owner j holds slots [j E_local, (j+1) E_local) in (expert, copy) order.
//   assign 4. the q-th assignment of expert e in ascending a = t k + slot goes to copy
//             q mod r_e.  q is the assignment's row inside its expert in the expert-
//             contiguous order of a one-owner dispatch layout.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

__global__ void eplb_assign_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ tok2row,
                                   const int32_t* __restrict__ expert_off, const int32_t* __restrict__ replica_off,
                                   const int32_t* __restrict__ replica_slots, int A, int E, int n_slots,
                                   int32_t* __restrict__ phys, int* status) {
  const int a = blockIdx.x * blockDim.x + threadIdx.x;
  if (a >= A) return;
  int e = ids[a];
  if (e == -1) {  // a dropped assignment stays dropped
    phys[a] = -1;
    return;
  }
  if (e < 0 || e >= E) {  // the layout pass counted it as expert 0 as well
    report(status, MOE_ERR_BAD_INDEX);
    e = 0;
  }
  const int q = tok2row[a] - expert_off[e];
  const int r0 = replica_off[e], r1 = replica_off[e + 1];
  int slot = 0;
  if (r0 < 0 || r1 <= r0 || r1 > n_slots) {
    report(status, MOE_ERR_BAD_INDEX);
  } else {
    slot = replica_slots[r0 + q % (r1 - r0)];
    if (slot < 0 || slot >= n_slots) {
      report(status, MOE_ERR_BAD_INDEX);
      slot = 0;
    }
  }
  phys[a] = slot;
}

// One-owner layout of the logical ids inside the caller's workspace.
struct EplbWs {
  moe_layout lay;
  void* scratch;
  size_t total;
};

static inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

static EplbWs carve_eplb(const moe_config& c, void* base) {
  const size_t A = (size_t)c.N * c.k;
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t n) {
    int32_t* r = reinterpret_cast<int32_t*>(p ? p + off : nullptr);
    off += al256(n * sizeof(int32_t));
    return r;
  };
  EplbWs w;
  w.lay.n_e = take(c.E);
  w.lay.expert_off = take(c.E + 1);
  w.lay.C = take(1);
  w.lay.send_off = take(1);
  w.lay.recv_off = take(2);
  w.lay.tok2send = take(A);
  w.lay.send2row = take(A);
  w.lay.ret2tok = take(A);
  w.lay.tok2row = take(A);
  w.lay.row2tok = take(A);
  w.lay.tile_off = take(c.E + 1);
  w.scratch = p ? p + off : nullptr;
  const int nchunks = A > 0 ? (int)((A + kLayoutChunk - 1) / kLayoutChunk) : 0;
  off += al256(layout_ws_bytes((int)A, c.E, 1, nchunks));
  w.total = off;
  return w;
}

static moe_config one_owner(const moe_config& c) {
  moe_config o = c;
  o.P = 1;
  o.n_shared = 0;
  return o;
}

size_t eplb_ws_bytes(const moe_config& c) { return carve_eplb(one_owner(c), nullptr).total; }

// Capacity ("ep_deepep" explainer §4): the q-th assignment of expert e (ascending a) is
// kept when q < capacity, else dropped (-1).  q comes from the same one-owner layout.
__global__ void capacity_keep_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ tok2row,
                                     const int32_t* __restrict__ expert_off, int A, int E, int capacity,
                                     int32_t* __restrict__ kept) {
  const int a = blockIdx.x * blockDim.x + threadIdx.x;
  if (a >= A) return;
  int e = ids[a];
  if (e == -1) {
    kept[a] = -1;
    return;
  }
  if (e < 0 || e >= E) e = 0;  // reported by the layout pass, counted as expert 0 there
  kept[a] = (tok2row[a] - expert_off[e] < capacity) ? e : -1;
}

cudaError_t launch_eplb_assign(const moe_config& c, const int32_t* ids, const int32_t* replica_off,
                               const int32_t* replica_slots, int n_slots, int32_t* phys, int32_t* status, void* ws,
                               cudaStream_t st) {
  const moe_config o = one_owner(c);
  EplbWs w = carve_eplb(o, ws);
  cudaError_t e = launch_layout(o, nullptr, ids, w.lay, status, w.scratch, st);
  if (e != cudaSuccess) return e;
  const int A = c.N * c.k;
  if (A == 0) return cudaSuccess;
  eplb_assign_kernel<<<(A + 255) / 256, 256, 0, st>>>(ids, w.lay.tok2row, w.lay.expert_off, replica_off,
                                                      replica_slots, A, c.E, n_slots, phys, status);
  return cudaGetLastError();
}

cudaError_t launch_capacity_keep(const moe_config& c, const int32_t* ids, int capacity, int32_t* kept,
                                 int32_t* status, void* ws, cudaStream_t st) {
  const moe_config o = one_owner(c);
  EplbWs w = carve_eplb(o, ws);
  cudaError_t e = launch_layout(o, nullptr, ids, w.lay, status, w.scratch, st);
  if (e != cudaSuccess) return e;
  const int A = c.N * c.k;
  if (A == 0) return cudaSuccess;
  capacity_keep_kernel<<<(A + 255) / 256, 256, 0, st>>>(ids, w.lay.tok2row, w.lay.expert_off, A, c.E, capacity,
                                                        kept);
  return cudaGetLastError();
}

// Steps 1-3 on the host (plain C++, exact integer arithmetic).
moe_status eplb_plan(int E, int R, int P, const int64_t* load, int32_t* copies, int32_t* replica_off,
                     int32_t* replica_slots, int32_t* slot_expert, int32_t* slot_owner, int64_t* owner_load) {
  const int S = E + R, per = S / P;
  std::vector<int64_t> r(E, 1);
  for (int x = 0; x < R; ++x) {  // step 1
    int best = 0;
    for (int e = 1; e < E; ++e)
      if (load[e] * r[best] > load[best] * r[e]) best = e;
    ++r[best];
  }
  struct Copy {
    int64_t rows;
    int e, c;
  };
  std::vector<Copy> cp;
  for (int e = 0; e < E; ++e)
    for (int c = 0; c < r[e]; ++c) cp.push_back({load[e] / r[e] + (c < load[e] % r[e] ? 1 : 0), e, c});
  std::sort(cp.begin(), cp.end(), [](const Copy& u, const Copy& v) {
    if (u.rows != v.rows) return u.rows > v.rows;
    if (u.e != v.e) return u.e < v.e;
    return u.c < v.c;
  });
  std::vector<int64_t> oload(P, 0);
  std::vector<int> room(P, per);
  std::vector<std::vector<char>> holds(P, std::vector<char>(E, 0));
  std::vector<int> owner_of_copy(S);  // indexed by replica_off[e] + c
  std::vector<int> off(E + 1, 0);
  for (int e = 0; e < E; ++e) off[e + 1] = off[e] + (int)r[e];
  for (const Copy& u : cp) {  // step 2
    int best = -1;
    for (int j = 0; j < P; ++j) {
      if (room[j] == 0) continue;
      if (best < 0) {
        best = j;
        continue;
      }
      const bool fj = !holds[j][u.e], fb = !holds[best][u.e];
      if (fj != fb) {
        if (fj) best = j;
        continue;
      }
      if (oload[j] < oload[best]) best = j;
    }
    owner_of_copy[off[u.e] + u.c] = best;
    oload[best] += u.rows;
    --room[best];
    holds[best][u.e] = 1;
  }
  std::vector<int> fill(P, 0);
  for (int e = 0; e < E; ++e) {  // step 3: (expert, copy) order inside each owner
    copies[e] = (int32_t)r[e];
    replica_off[e] = off[e];
    for (int c = 0; c < r[e]; ++c) {
      const int j = owner_of_copy[off[e] + c];
      const int slot = j * per + fill[j]++;
      slot_expert[slot] = e;
      slot_owner[slot] = j;
      replica_slots[off[e] + c] = slot;
    }
  }
  replica_off[E] = off[E];
  for (int j = 0; j < P; ++j) owner_load[j] = oload[j];
  return MOE_OK;
}

}  // namespace moe
