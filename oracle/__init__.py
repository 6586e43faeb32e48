"""CPU oracle for the deterministic MoE layer, forward and backward (test infrastructure only).

Only the test suite, the package smoke check and the benchmark's CPU-baseline
leg may import this package. It wraps oracle/moe_oracle.cpp (plain C++,
OpenMP) through ctypes and orchestrates its steps with plain numpy; it shares
no code with the CUDA library.

Parity pins: every function here is checked in tests/ against something other
than itself (brute force, closed forms, library routines, the pages' worked
numbers). The design notes list them; no function is left unpinned.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_route_topk.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                        _i32p, _f32p, _f64p]
        L.oracle_route_topk.restype = ctypes.c_int
        L.oracle_schedule.argtypes = [_i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, _i32p, _i32p,
                                      _i32p, _i32p, _i64p]
        L.oracle_schedule.restype = ctypes.c_int
        L.oracle_place_closed_form.argtypes = [_i32p] + [ctypes.c_int32] * 5 + [_i32p, _i32p]
        L.oracle_place_closed_form.restype = ctypes.c_int
        L.oracle_place_queue_sim.argtypes = [_i32p] + [ctypes.c_int32] * 5 + [ctypes.c_int64, _i32p,
                                                                               _i32p, _i32p]
        L.oracle_place_queue_sim.restype = ctypes.c_int
        L.oracle_wave_floor.argtypes = [ctypes.c_int64] * 3
        L.oracle_wave_floor.restype = ctypes.c_int64
        L.oracle_dispatch_rows.argtypes = [_u16p, ctypes.c_int32, ctypes.c_int32, _i32p, _i64p,
                                           ctypes.c_int64, _u16p]
        L.oracle_dispatch_rows.restype = None
        ptr_arr = ctypes.POINTER(ctypes.c_void_p)
        L.oracle_ffn_rows.argtypes = [_u16p, ctypes.c_int64, _i32p, ctypes.c_int32, ctypes.c_int32,
                                      ptr_arr, ptr_arr, ptr_arr, _u16p, _f64p]
        L.oracle_ffn_rows.restype = None
        L.oracle_combine_f64.argtypes = [_f64p, ctypes.c_int32, _i64p, _f64p, ctypes.c_int64,
                                         ctypes.c_int32, _f64p, _u16p]
        L.oracle_combine_f64.restype = None
        L.oracle_combine_f32.argtypes = [_f32p, ctypes.c_int32, _i64p, _f32p, ctypes.c_int64,
                                         ctypes.c_int32, _u16p]
        L.oracle_ffn_bwd_rows.argtypes = [_u16p, _u16p, _f64p, ctypes.c_int64, _i32p, ctypes.c_int32,
                                          ctypes.c_int32, ptr_arr, ptr_arr, ptr_arr, ctypes.c_int,
                                          _f64p, _f64p, _u16p, _u16p, _u16p]
        L.oracle_ffn_bwd_rows.restype = None
        L.oracle_wgrad_expert.argtypes = [_u16p, _u16p, _f64p, ctypes.c_int64, ctypes.c_int32,
                                          ctypes.c_int32, _u16p, _u16p, _u16p, _i32p, ctypes.c_int32,
                                          _i32p, ctypes.c_int32, ctypes.c_int, _f64p, _f64p, _f64p]
        L.oracle_wgrad_expert.restype = None
        L.oracle_router_bwd.argtypes = [_f64p, _f64p, _i32p, ctypes.c_int64, ctypes.c_int32,
                                        ctypes.c_int32, _f64p]
        L.oracle_router_bwd.restype = None
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_mx_quantize.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int32, _u8p, _u8p]
        L.oracle_mx_quantize.restype = None
        L.oracle_mx_dequantize.argtypes = [_u8p, _u8p, ctypes.c_int64, ctypes.c_int32, _f64p]
        L.oracle_mx_dequantize.restype = None
        L.oracle_combine_f32.restype = None
        L.oracle_round_bf16.argtypes = [ctypes.c_double]
        L.oracle_round_bf16.restype = ctypes.c_uint16
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _p(a: np.ndarray, t):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(t)


def _np(x, dtype):
    """torch tensor or array-like -> contiguous numpy array of dtype (CPU)."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            x = x.view(torch.int16)
        x = x.numpy()
    a = np.asarray(x)
    dt = np.dtype(dtype)
    if a.dtype != dt and a.dtype.kind in "iu" and dt.kind in "iu" and a.dtype.itemsize == dt.itemsize:
        a = a.view(dt)  # reinterpret bits (bf16 / int16 -> uint16)
    return np.ascontiguousarray(a, dtype=dt)


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def round_bf16(v: float) -> int:
    return int(lib().oracle_round_bf16(float(v)))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rows_cap(P: int, N: int, k: int, E: int, pad: int) -> int:
    """Upper bound on padded rows: every route, plus at most pad-1 padding rows per expert."""
    return P * N * k + E * (pad - 1)


def route_topk(logits, k: int):
    """ids int32 [T,k], gates fp32 [T,k], gates fp64 [T,k] (top-k by logit desc, id asc)."""
    lg = _np(logits, np.float32)
    T, E = lg.shape
    ids = np.zeros((T, k), np.int32)
    g32 = np.zeros((T, k), np.float32)
    g64 = np.zeros((T, k), np.float64)
    rc = lib().oracle_route_topk(_p(lg, _f32p), T, E, k, _p(ids, _i32p), _p(g32, _f32p),
                                 _p(g64, _f64p))
    if rc:
        raise ValueError(f"oracle_route_topk rc={rc}")
    return ids, g32, g64


def schedule(ids, P: int, N: int, k: int, E: int, pad: int = 256):
    """Counting-sort schedule. Returns dict(phi [rows,2], offsets [E+1], counts [E,P],
    route_row [P,N,k], reads, counter_words, threads)."""
    idn = _np(ids, np.int32).reshape(-1)
    cap = max(rows_cap(P, N, k, E, pad), 1)
    phi = np.full((cap, 2), -7, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    counts = np.zeros((E, P), np.int32)
    rr = np.zeros((P, N, k), np.int32)
    stats = np.zeros(3, np.int64)
    rc = lib().oracle_schedule(_p(idn, _i32p), P, N, k, E, pad, cap, _p(phi, _i32p),
                               _p(offsets, _i32p), _p(counts, _i32p), _p(rr, _i32p),
                               _p(stats, _i64p))
    if rc:
        raise ValueError(f"oracle_schedule rc={rc}")
    rows = int(offsets[E])
    return dict(phi=phi[:rows].copy(), offsets=offsets, counts=counts, route_row=rr,
                reads=int(stats[0]), counter_words=int(stats[1]), threads=int(stats[2]))


def place_closed_form(ids, P: int, N: int, k: int, E: int, pad: int = 256):
    idn = _np(ids, np.int32).reshape(-1)
    offsets = np.zeros(E + 1, np.int32)
    rr = np.zeros((P, N, k), np.int32)
    rc = lib().oracle_place_closed_form(_p(idn, _i32p), P, N, k, E, pad, _p(offsets, _i32p),
                                        _p(rr, _i32p))
    if rc:
        raise ValueError(f"oracle_place_closed_form rc={rc}")
    return offsets, rr


def place_queue_sim(ids, P: int, N: int, k: int, E: int, pad: int = 256):
    idn = _np(ids, np.int32).reshape(-1)
    cap = max(rows_cap(P, N, k, E, pad), 1)
    offsets = np.zeros(E + 1, np.int32)
    rr = np.zeros((P, N, k), np.int32)
    phi = np.full((cap, 2), -7, np.int32)
    rc = lib().oracle_place_queue_sim(_p(idn, _i32p), P, N, k, E, pad, cap, _p(offsets, _i32p),
                                      _p(rr, _i32p), _p(phi, _i32p))
    if rc:
        raise ValueError(f"oracle_place_queue_sim rc={rc}")
    return offsets, rr, phi[: int(offsets[E])].copy()


def wave_floor(H: int, I: int, C: int) -> int:
    return int(lib().oracle_wave_floor(H, I, C))


def dispatch_rows(x_bits: np.ndarray, N: int, phi: np.ndarray, rows) -> np.ndarray:
    """Gather rows of Phi from x ([P*N, H] bf16 bits) -> [n, H] bf16 bits."""
    xb = _np(x_bits, np.uint16)
    H = xb.shape[1]
    phn = np.ascontiguousarray(phi, np.int32)
    rws = np.ascontiguousarray(np.asarray(rows, np.int64))
    out = np.zeros((len(rws), H), np.uint16)
    lib().oracle_dispatch_rows(_p(xb, _u16p), N, H, _p(phn, _i32p), _p(rws, _i64p), len(rws),
                               _p(out, _u16p))
    return out


def ffn_rows(xg_bits: np.ndarray, experts, W1: dict, W3: dict, W2: dict, H: int, I: int):
    """SwiGLU FFN of rows xg_bits [n,H] (bf16 bits) with per-row experts.

    W1/W3/W2 map expert id -> numpy uint16 arrays [H,I] / [H,I] / [I,H].
    Returns h bf16 bits [n,I] and y fp64 [n,H].
    """
    xb = np.ascontiguousarray(xg_bits, np.uint16)
    ex = np.ascontiguousarray(np.asarray(experts, np.int32))
    n = len(ex)
    E = int(ex.max()) + 1 if n else 1
    keep = []
    arrs = []
    for Wd in (W1, W3, W2):
        a = (ctypes.c_void_p * E)()
        for e, w in Wd.items():
            if e < E:
                w = np.ascontiguousarray(w, np.uint16)
                keep.append(w)
                a[e] = w.ctypes.data
        arrs.append(a)
    for e in set(ex.tolist()):
        if not (arrs[0][e] and arrs[1][e] and arrs[2][e]):
            raise ValueError(f"weights of expert {e} not given")
    h = np.zeros((n, I), np.uint16)
    y = np.zeros((n, H), np.float64)
    if n:
        lib().oracle_ffn_rows(_p(xb, _u16p), n, _p(ex, _i32p), H, I,
                              ctypes.cast(arrs[0], ctypes.POINTER(ctypes.c_void_p)),
                              ctypes.cast(arrs[1], ctypes.POINTER(ctypes.c_void_p)),
                              ctypes.cast(arrs[2], ctypes.POINTER(ctypes.c_void_p)),
                              _p(h, _u16p), _p(y, _f64p))
    return h, y


def combine_f64(y: np.ndarray, sel, g, k: int):
    """out[a] = sum_j g[a,j] * y[sel[a,j]] (fp64). Returns (out64, out_bf16_bits)."""
    yy = np.ascontiguousarray(y, np.float64)
    H = yy.shape[1]
    s = np.ascontiguousarray(np.asarray(sel, np.int64).reshape(-1))
    gg = np.ascontiguousarray(np.asarray(g, np.float64).reshape(-1))
    n = len(s) // k
    out64 = np.zeros((n, H), np.float64)
    outb = np.zeros((n, H), np.uint16)
    lib().oracle_combine_f64(_p(yy, _f64p), H, _p(s, _i64p), _p(gg, _f64p), n, k, _p(out64, _f64p),
                             _p(outb, _u16p))
    return out64, outb


def combine_f32(y: np.ndarray, sel, g, k: int) -> np.ndarray:
    """Fixed-order fp32 combine (fmaf, ascending slot) -> bf16 bits [n, H]."""
    yy = np.ascontiguousarray(y, np.float32)
    H = yy.shape[1]
    s = np.ascontiguousarray(np.asarray(sel, np.int64).reshape(-1))
    gg = np.ascontiguousarray(np.asarray(g, np.float32).reshape(-1))
    n = len(s) // k
    outb = np.zeros((n, H), np.uint16)
    lib().oracle_combine_f32(_p(yy, _f32p), H, _p(s, _i64p), _p(gg, _f32p), n, k, _p(outb, _u16p))
    return outb


def expert_of_rows(offsets: np.ndarray, rows) -> np.ndarray:
    """Expert l of each row: the segment with offsets[l] <= row < offsets[l+1]."""
    off = np.asarray(offsets, np.int64)
    return (np.searchsorted(off, np.asarray(rows, np.int64), side="right") - 1).astype(np.int32)


def layer_tokens(logits, x_bits, weights, P: int, N: int, k: int, E: int, H: int, I: int,
                 tokens, pad: int = 256, experts_per_group: int = 32):
    """The whole layer for a set of tokens: route all tokens, schedule all routes,
    then dispatch, FFN and combine only the rows the chosen tokens need.

    weights: (W1, W3, W2) dicts expert -> numpy uint16 arrays (only the experts
    the chosen tokens use need to be present), or a callable that returns
    such dicts for a list of experts; the FFN then runs over groups of
    `experts_per_group` experts at a time, so only one group's weights are
    held in host memory at once.
    Returns dict with ids, gates32, gates64, sched, out64 [n,H], out_bf16 [n,H],
    y rows per (token, slot) and h rows.
    """
    ids, g32, g64 = route_topk(logits, k)
    sch = schedule(ids.reshape(P, N, k), P, N, k, E, pad)
    toks = np.asarray(tokens, np.int64)
    rr = sch["route_row"].reshape(P * N, k)
    sel_rows = rr[toks].reshape(-1).astype(np.int64)
    uniq, inv = np.unique(sel_rows, return_inverse=True)
    xg = dispatch_rows(x_bits, N, sch["phi"], uniq)
    ex = expert_of_rows(sch["offsets"], uniq)
    if callable(weights):
        h = np.zeros((len(uniq), I), np.uint16)
        y = np.zeros((len(uniq), H), np.float64)
        used = np.unique(ex)
        for g0 in range(0, len(used), experts_per_group):
            grp = used[g0:g0 + experts_per_group]
            m = np.isin(ex, grp)
            h[m], y[m] = ffn_rows(xg[m], ex[m], *weights(grp.tolist()), H=H, I=I)
    else:
        h, y = ffn_rows(xg, ex, *weights, H=H, I=I)
    out64, outb = combine_f64(y, inv.reshape(len(toks), k), g64[toks], k)
    return dict(ids=ids, gates32=g32, gates64=g64, sched=sch, out64=out64, out_bf16=outb,
                rows=uniq, row_index=inv.reshape(len(toks), k), xg=xg, h=h, y=y,
                experts=ex)


# ---------------------------------------------------------------- backward
def _weight_ptr_arrays(experts, W1: dict, W3: dict, W2: dict):
    ex = np.asarray(experts, np.int32)
    E = int(ex.max()) + 1 if len(ex) else 1
    keep, arrs = [], []
    for Wd in (W1, W3, W2):
        a = (ctypes.c_void_p * E)()
        for e, w in Wd.items():
            if e < E:
                w = np.ascontiguousarray(w, np.uint16)
                keep.append(w)
                a[e] = w.ctypes.data
        arrs.append(a)
    for e in set(ex.tolist()):
        if not (arrs[0][e] and arrs[1][e] and arrs[2][e]):
            raise ValueError(f"weights of expert {e} not given")
    return keep, [ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p)) for a in arrs]


def ffn_bwd_rows(xg_bits, dys_bits, g, experts, W1: dict, W3: dict, W2: dict, H: int, I: int,
                 exact: bool = False):
    """Backward through the SwiGLU expert FFN, one route row at a time.

    xg_bits/dys_bits [n,H] bf16 bits (the row's token activations and upstream
    gradient), g [n] gates, experts [n]. Returns dict dgate [n] (fp64),
    dxg [n,H] (fp64) and, unless exact, da/db/hg [n,I] bf16 bits.
    """
    xb = np.ascontiguousarray(xg_bits, np.uint16)
    db_ = np.ascontiguousarray(dys_bits, np.uint16)
    gg = np.ascontiguousarray(np.asarray(g, np.float64).reshape(-1))
    ex = np.ascontiguousarray(np.asarray(experts, np.int32))
    n = len(ex)
    out = dict(dgate=np.zeros(n, np.float64), dxg=np.zeros((n, H), np.float64),
               da=np.zeros((n, I), np.uint16), db=np.zeros((n, I), np.uint16),
               hg=np.zeros((n, I), np.uint16))
    if n:
        keep, arrs = _weight_ptr_arrays(ex, W1, W3, W2)
        lib().oracle_ffn_bwd_rows(_p(xb, _u16p), _p(db_, _u16p), _p(gg, _f64p), n, _p(ex, _i32p),
                                  H, I, *arrs, int(bool(exact)), _p(out["dgate"], _f64p),
                                  _p(out["dxg"], _f64p), _p(out["da"], _u16p),
                                  _p(out["db"], _u16p), _p(out["hg"], _u16p))
    if exact:
        for key in ("da", "db", "hg"):
            del out[key]
    return out


def wgrad_expert(xg_bits, dys_bits, g, W1e, W3e, W2e, hs, is_, exact: bool = False):
    """Weight gradients of one expert from all R rows it received, at the chosen
    columns: dW1[hs][:, is_], dW3[hs][:, is_] ([n_h, n_i]) and dW2[is_][:, hs]
    ([n_i, n_h]), fp64."""
    xb = np.ascontiguousarray(xg_bits, np.uint16)
    db_ = np.ascontiguousarray(dys_bits, np.uint16)
    gg = np.ascontiguousarray(np.asarray(g, np.float64).reshape(-1))
    R, H = xb.shape if xb.size else (0, np.asarray(W2e).shape[1])
    I = np.asarray(W1e).shape[1]
    hh = np.ascontiguousarray(np.asarray(hs, np.int32))
    ii = np.ascontiguousarray(np.asarray(is_, np.int32))
    w1, w3, w2 = (np.ascontiguousarray(w, np.uint16) for w in (W1e, W3e, W2e))
    dW1 = np.zeros((len(hh), len(ii)), np.float64)
    dW3 = np.zeros((len(hh), len(ii)), np.float64)
    dW2 = np.zeros((len(ii), len(hh)), np.float64)
    lib().oracle_wgrad_expert(_p(xb, _u16p) if R else _p(np.zeros(1, np.uint16), _u16p),
                              _p(db_, _u16p) if R else _p(np.zeros(1, np.uint16), _u16p),
                              _p(gg, _f64p) if R else _p(np.zeros(1), _f64p), R, H, I,
                              _p(w1, _u16p), _p(w3, _u16p), _p(w2, _u16p), _p(hh, _i32p), len(hh),
                              _p(ii, _i32p), len(ii), int(bool(exact)), _p(dW1, _f64p),
                              _p(dW3, _f64p), _p(dW2, _f64p))
    return dW1, dW3, dW2


def router_bwd(dgate, g, ids, E: int) -> np.ndarray:
    """dlogits [n,E]: g_j (dgate_j - sum_j' g_j' dgate_j') at the chosen experts, 0 elsewhere."""
    dg = np.ascontiguousarray(np.asarray(dgate, np.float64))
    gg = np.ascontiguousarray(np.asarray(g, np.float64))
    ii = np.ascontiguousarray(np.asarray(ids, np.int32))
    n, k = ii.shape
    out = np.zeros((n, E), np.float64)
    if n:
        lib().oracle_router_bwd(_p(dg, _f64p), _p(gg, _f64p), _p(ii, _i32p), n, k, E, _p(out, _f64p))
    return out


def layer_backward_tokens(logits, x_bits, dout_bits, weights, k: int, E: int, H: int, I: int,
                          tokens, exact: bool = False):
    """Gradients of the layer for a set of tokens: dx [n,H] (fp64, before the
    bf16 cast), dlogits [n,E] and the gate gradients dgate [n,k].

    Each route (t, j) is one expert row: its token's activations x[t] and
    upstream gradient dout[t], gate g[t,j] (the fp64 softmax over the chosen
    logits) and expert ids[t,j]. The push-reverse-dispatch sums a token's k
    row gradients in ascending slot order.
    """
    ids, g32, g64 = route_topk(logits, k)
    toks = np.asarray(list(tokens), np.int64)
    n = len(toks)
    xb = np.asarray(x_bits, np.uint16)[toks]
    db_ = np.asarray(dout_bits, np.uint16)[toks]
    rx = np.repeat(xb, k, axis=0)
    rd = np.repeat(db_, k, axis=0)
    ex = ids[toks].reshape(-1)
    r = ffn_bwd_rows(rx, rd, g64[toks].reshape(-1), ex, *weights, H=H, I=I, exact=exact)
    dxg = r["dxg"].reshape(n, k, H)
    dx = np.zeros((n, H), np.float64)
    for j in range(k):
        dx += dxg[:, j, :]
    dgate = r["dgate"].reshape(n, k)
    dlogits = router_bwd(dgate, g64[toks], ids[toks], E)
    return dict(ids=ids, gates32=g32, gates64=g64, dx64=dx, dgate=dgate, dlogits=dlogits,
                rows=r)


def wgrad_sample(logits, x_bits, dout_bits, weights, k: int, E: int, experts, hs, is_,
                 exact: bool = False):
    """dW1/dW3 [n_h, n_i] and dW2 [n_i, n_h] at the chosen columns for each chosen
    expert: {e: (dW1s, dW3s, dW2s)}. An expert's rows are every route that chose
    it (token activations, upstream gradient and gate of the route)."""
    ids, _, g64 = route_topk(logits, k)
    xb = np.asarray(x_bits, np.uint16)
    db_ = np.asarray(dout_bits, np.uint16)
    W1, W3, W2 = weights
    out = {}
    for e in experts:
        t, j = np.nonzero(ids == e)
        out[e] = wgrad_expert(xb[t], db_[t], g64[t, j], W1[e], W3[e], W2[e], hs, is_, exact)
    return out


# ---------------------------------------------------------------- MXFP8
def e4m3_value(codes) -> np.ndarray:
    """float64 values of E4M3 codes (NaN for S.1111.111)."""
    c = np.asarray(codes, np.uint8)
    return np.array([lib().oracle_e4m3_value(int(x)) for x in c.reshape(-1)]).reshape(c.shape)


def e4m3_encode(values) -> np.ndarray:
    """E4M3 codes of values: nearest, ties to even, magnitudes above 448 clamped."""
    v = np.asarray(values, np.float64)
    return np.array([lib().oracle_e4m3_encode(float(x)) for x in v.reshape(-1)],
                    np.uint8).reshape(v.shape)


def mx_quantize(values):
    """MX (E4M3, blocks of 32 along the last axis): (codes [..., K], scales [..., K/32])."""
    v = np.ascontiguousarray(np.asarray(values, np.float64))
    K = v.shape[-1]
    if K % 32:
        raise ValueError("the last axis must be a multiple of 32")
    n = v.size // K
    q = np.zeros(v.shape, np.uint8)
    s = np.zeros(v.shape[:-1] + (K // 32,), np.uint8)
    if n:
        lib().oracle_mx_quantize(_p(v, _f64p), n, K, _p(q, _u8p), _p(s, _u8p))
    return q, s


def mx_dequantize(q, s) -> np.ndarray:
    qq = np.ascontiguousarray(np.asarray(q, np.uint8))
    ss = np.ascontiguousarray(np.asarray(s, np.uint8))
    K = qq.shape[-1]
    n = qq.size // K
    out = np.zeros(qq.shape, np.float64)
    if n:
        lib().oracle_mx_dequantize(_p(qq, _u8p), _p(ss, _u8p), n, K, _p(out, _f64p))
    return out


def mx_round(values, axis: int = -1) -> np.ndarray:
    """The values an MXFP8 operand stands for: quantised in blocks of 32 along
    `axis` (the GEMM's reduction dimension), then dequantised."""
    v = np.moveaxis(np.asarray(values, np.float64), axis, -1)
    q, s = mx_quantize(v)
    return np.moveaxis(mx_dequantize(q, s), -1, axis)


def _bits_f64(b) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def layer_tokens_mxfp8(logits, x_bits, weights, k: int, H: int, I: int, tokens, shared=None):
    """The layer with MXFP8 routed experts ("Mixture-of-Kittens", section 5),
    for a set of tokens: every GEMM operand is MX-quantised along its reduction
    dimension -- x rows along H, W1/W3 along H (per column i), h rows along I,
    W2 along I (per column) -- and the products, SwiGLU and combine run in
    fp64 on the values the quantised operands stand for:
      a = mx(x).mx(W1), b = mx(x).mx(W3), h = silu(a) * b,
      y = mx(h).mx(W2), out[t] = sum_j g_j y_j (gates: fp64 softmax of the top k).
    h is rounded to fp32 before its quantisation: the codes and scales are
    decided in the precision the kernels hold h in (the pages fix none).
    shared: None, or the bf16 shared expert's (Ws1 [H, I], Ws3 [H, I], Ws2
    [I, H]) bit patterns; its output, the bf16 FFN of x[t] (ffn_rows), is
    added to every token: out[t] += y_shared[t].
    Returns dict out64 [n, H], ids, gates64."""
    ids, g32, g64 = route_topk(logits, k)
    toks = np.asarray(list(tokens), np.int64)
    W1, W3, W2 = weights
    cache = {}

    def expert(e):
        if e not in cache:
            cache[e] = (mx_round(_bits_f64(W1[e]), axis=0), mx_round(_bits_f64(W3[e]), axis=0),
                        mx_round(_bits_f64(W2[e]), axis=0))
        return cache[e]

    xb = np.asarray(x_bits, np.uint16)
    out = np.zeros((len(toks), H), np.float64)
    for a_i, t in enumerate(toks):
        xt = mx_round(_bits_f64(xb[t]))
        for j in range(k):
            w1, w3, w2 = expert(int(ids[t, j]))
            a = xt @ w1
            b = xt @ w3
            h = (a / (1.0 + np.exp(-a)) * b).astype(np.float32).astype(np.float64)
            out[a_i] += g64[t, j] * (mx_round(h) @ w2)
    if shared is not None and len(toks):
        Ws1, Ws3, Ws2 = shared
        _, ys = ffn_rows(xb[toks], np.zeros(len(toks), np.int32), {0: Ws1}, {0: Ws3}, {0: Ws2},
                         H, I)
        out += ys
    return dict(out64=out, ids=ids, gates64=g64)


def ffn_rows_mxfp8(xg_bits, experts, W1: dict, W3: dict, W2: dict, H: int, I: int):
    """The SwiGLU expert FFN with MXFP8 operands ("Mixture-of-Kittens",
    section 5) for gathered rows xg_bits [n, H] (bf16 bits) with per-row
    experts. Every GEMM operand is MX-quantised along its reduction dimension
    and the arithmetic runs in fp64 on the values the codes stand for:
      a = mx(x).mx(W1), b = mx(x).mx(W3), h = silu(a) * b,
      (hq, hs) = the MX codes and scales of h (blocks of 32 along I), decided
      on h rounded to fp32, the precision the kernel holds h in,
      y = dq(hq, hs).mx(W2).
    W1/W3/W2 map expert id -> uint16 [H, I] / [H, I] / [I, H].
    Returns hq uint8 [n, I], hs uint8 [n, I/32] (row-major), y fp64 [n, H]."""
    xb = np.asarray(xg_bits, np.uint16)
    ex = np.asarray(experts, np.int64)
    n = len(ex)
    hq = np.zeros((n, I), np.uint8)
    hs = np.zeros((n, I // 32), np.uint8)
    y = np.zeros((n, H), np.float64)
    for e in np.unique(ex):
        rows = np.nonzero(ex == e)[0]
        xr = mx_round(_bits_f64(xb[rows]))
        w1 = mx_round(_bits_f64(W1[int(e)]), axis=0)
        w3 = mx_round(_bits_f64(W3[int(e)]), axis=0)
        w2 = mx_round(_bits_f64(W2[int(e)]), axis=0)
        a = xr @ w1
        b = xr @ w3
        with np.errstate(over="ignore"):
            h = (a / (1.0 + np.exp(-a)) * b).astype(np.float32).astype(np.float64)
        q, s = mx_quantize(h)
        hq[rows], hs[rows] = q, s
        y[rows] = mx_dequantize(q, s) @ w2
    return hq, hs, y
