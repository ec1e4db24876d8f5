// Appending one token per (batch, kv-head) unit at position pos: the new K and V rows go into
// the tail window's page (a page is popped from the unit's free stack when the token starts a
// page), the V row also into the tail window's V staging area (for its norms when the window
// completes), and a token that starts a window opens it as the tail ("Resumo Técnico: QEvict",
// Declaração do Problema: the cache grows by one token per decode step).
#pragma once
#include "qe_internal.cuh"

// Run by every thread of one CTA (at least D/8 threads) for unit u; s_page is a shared int.
// Ends with a barrier; the rows are then visible to the CTA's later bulk copies.
__device__ __forceinline__ void append_token(const DevState& st, int u, int pos, const uint4* k_new,
                                             const uint4* v_new, uint4* tailV, int* s_page) {
  const int b = u / st.Hkv, kvh = u % st.Hkv;
  const int w = st.window, tw = pos / w, t = pos % w, pg = t / QE_PAGE, r = pos % QE_PAGE;
  const int vpr = st.D * 2 / 16;
  // the new rows do not depend on the page lookup: load them first
  uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
  if (threadIdx.x < vpr) {
    kv = k_new[(size_t)u * vpr + threadIdx.x];
    vv = v_new[(size_t)u * vpr + threadIdx.x];
  }
  if (threadIdx.x == 0) {
    const size_t wi = (size_t)u * st.Wmax + tw;
    int page = -1;
    if (t == 0) {
      st.win_tier[wi] = QE_TIER_TAIL;
      st.win_slot[wi] = -1;
      st.mass[wi] = 0.f;
      st.pert[wi] = 0.f;
    }
    if (r == 0) {
      const int top = st.stacks[u * 4 + 0];
      if (top <= 0) {
        qe_record_error(st.status, QE_ERR_POOL_EXHAUSTED, u);
      } else {
        page = st.page_free[(size_t)u * st.P + top - 1];
        st.stacks[u * 4 + 0] = top - 1;
        st.win_pages[wi * st.ppw + pg] = page;
      }
    } else {
      page = st.win_pages[wi * st.ppw + pg];
    }
    if (page >= st.P) {
      qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
      page = -1;
    }
    *s_page = page;
  }
  __syncthreads();
  if (t == 0)
    for (int i = threadIdx.x; i < w * st.G; i += blockDim.x) st.tail_p[(size_t)u * w * st.G + i] = 0.f;
  const int page = *s_page;
  if (page >= 0 && threadIdx.x < vpr) {
    uint4* base = reinterpret_cast<uint4*>(st.pages + ((size_t)u * st.P + page) * st.page_bytes);
    const int c = threadIdx.x;
    base[r * vpr + c] = kv;
    base[(QE_PAGE + r) * vpr + c] = vv;
    tailV[(((size_t)kvh * st.B + b) * w + t) * vpr + c] = vv;
  }
  // order these generic-proxy writes before async-proxy (bulk copy) reads of the same memory
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __syncthreads();
}

// The same append run by one warp (lanes 0..31, D/8 <= 32), synchronising the warp only.
// Returns (in every lane) the page that received the token, -1 if none could be taken.
__device__ __forceinline__ int append_token_warp(const DevState& st, int u, int pos, const uint4* k_new,
                                                  const uint4* v_new, uint4* tailV) {
  const int lane = threadIdx.x & 31;
  const int b = u / st.Hkv, kvh = u % st.Hkv;
  const int w = st.window, tw = pos / w, t = pos % w, pg = t / QE_PAGE, r = pos % QE_PAGE;
  const int vpr = st.D * 2 / 16;
  uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
  if (lane < vpr) {
    kv = k_new[(size_t)u * vpr + lane];
    vv = v_new[(size_t)u * vpr + lane];
  }
  int page = -1;
  if (lane == 0) {
    const size_t wi = (size_t)u * st.Wmax + tw;
    if (t == 0) {
      st.win_tier[wi] = QE_TIER_TAIL;
      st.win_slot[wi] = -1;
      st.mass[wi] = 0.f;
      st.pert[wi] = 0.f;
    }
    if (r == 0) {
      const int top = st.stacks[u * 4 + 0];
      if (top <= 0) {
        qe_record_error(st.status, QE_ERR_POOL_EXHAUSTED, u);
      } else {
        page = st.page_free[(size_t)u * st.P + top - 1];
        st.stacks[u * 4 + 0] = top - 1;
        st.win_pages[wi * st.ppw + pg] = page;
      }
    } else {
      page = st.win_pages[wi * st.ppw + pg];
    }
    if (page >= st.P) {
      qe_record_error(st.status, QE_ERR_DEVICE_FAULT, u);
      page = -1;
    }
  }
  page = __shfl_sync(0xffffffffu, page, 0);
  if (t == 0)
    for (int i = lane; i < w * st.G; i += 32) st.tail_p[(size_t)u * w * st.G + i] = 0.f;
  if (page >= 0 && lane < vpr) {
    uint4* base = reinterpret_cast<uint4*>(st.pages + ((size_t)u * st.P + page) * st.page_bytes);
    base[r * vpr + lane] = kv;
    base[(QE_PAGE + r) * vpr + lane] = vv;
    tailV[(((size_t)kvh * st.B + b) * w + t) * vpr + lane] = vv;
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __syncwarp();
  return page;
}
