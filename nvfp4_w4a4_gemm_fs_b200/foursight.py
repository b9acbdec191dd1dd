"""Thin torch-tensor wrappers with the names of the C ABI (argument marshalling only).

All tensors must already live on the current CUDA device; outputs are caller-allocated
(helpers ``alloc_*`` allocate them with torch, outside any timed or captured region).
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _lib
from ._lib import FS_DTYPE_BF16, FS_DTYPE_F32, check

__all__ = [
    "fs_channel_stats", "fs_stats_check", "fs_select_topk", "fs_prepare_weights",
    "fs_quantize_splice", "fs_quantize_splice_grouped", "fs_quantize_splice_stats", "fs_splice_gemm", "fs_splice_gemm_grouped",
    "fs_seq_filter", "Plan", "StatsState", "Packed", "side_cols", "sf_bytes", "grouped_rows", "compact_cols",
    "fs_splice_gemm_segmented", "fs_decode_splice_gemm", "stacked_packed", "fs_gemm_bf16", "fs_transpose_bf16", "fs_ste_backward",
    "fs_grpo_objective", "fs_k3_kl",
    "alloc_packed", "stream_handle", "ArgumentError",
]


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def stream_handle(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FS_DTYPE_BF16
    if t.dtype == torch.float32:
        return FS_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def side_cols(p: int) -> int:
    return _lib.load().fs_side_cols(p)


def sf_bytes(rows: int, K: int) -> int:
    return _lib.load().fs_sf_bytes(rows, K)


def grouped_rows(max_rows: int, E: int) -> int:
    return _lib.load().fs_grouped_rows(max_rows, E)


class StatsState:
    """Device state of fs_channel_stats for nprob input groups that share K."""

    def __init__(self, nprob: int, K: int, device="cuda"):
        self.nprob, self.K = nprob, K
        self.n = torch.zeros(nprob, dtype=torch.int64, device=device)
        self.s1 = torch.zeros(nprob, K, dtype=torch.int64, device=device)
        self.s2 = torch.zeros(nprob, K, dtype=torch.int64, device=device)
        self.amax = torch.zeros(nprob, K, dtype=torch.int32, device=device)
        self.flags = torch.zeros(nprob, dtype=torch.int32, device=device)

    def group(self, i: int):
        return self.n[i:i + 1], self.s1[i], self.s2[i], self.amax[i], self.flags[i:i + 1]

    _FIELDS = (("n", torch.int64), ("s1", torch.int64), ("s2", torch.int64), ("amax", torch.int32),
               ("flags", torch.int32))

    def state_dict(self) -> dict:
        """A checkpoint of the state as host tensors.  The moments are integer sums, so a state
        restored with load_state_dict continues bit-exactly where it stopped (row subsampling
        restarts at row 0 of each call, as it does without a checkpoint)."""
        d = {name: getattr(self, name).detach().to("cpu", copy=True) for name, _ in self._FIELDS}
        d["K"], d["nprob"] = self.K, self.nprob
        return d

    def load_state_dict(self, d: dict) -> None:
        """Restores a checkpoint taken from a state of the same nprob and K (any device)."""
        who = "StatsState.load_state_dict"
        _need(d.get("K") == self.K and d.get("nprob") == self.nprob, who,
              f"checkpoint of nprob={d.get('nprob')}, K={d.get('K')} for a state of nprob={self.nprob}, K={self.K}")
        for name, dtype in self._FIELDS:
            src, dst = d.get(name), getattr(self, name)
            _need(isinstance(src, torch.Tensor) and src.dtype == dtype and tuple(src.shape) == tuple(dst.shape), who,
                  f"field {name} must be {dtype} of shape {tuple(dst.shape)}")
        for name, _ in self._FIELDS:
            getattr(self, name).copy_(d[name])


class Packed:
    """Packed NVFP4 operand: q [R,K/2] u8, sf (tiled) u8, side [R,Pp] bf16."""

    def __init__(self, q, sf, side, rows, K, p):
        self.q, self.sf, self.side, self.rows, self.K, self.p = q, sf, side, rows, K, p


def alloc_packed(rows: int, K: int, p: int, device="cuda") -> Packed:
    pp = side_cols(p)
    q = torch.empty(max(rows, 1), K // 2, dtype=torch.uint8, device=device)
    sf = torch.empty(sf_bytes(rows, K), dtype=torch.uint8, device=device)
    side = torch.empty(max(rows, 1), max(pp, 8), dtype=torch.bfloat16, device=device)[:, :pp]
    return Packed(q, sf, side if pp else side, rows, K, p)


# ------------------------------------------------------------------ extents the C ABI cannot see
# The library takes plain pointers, so it cannot tell how many bytes stand behind them; these
# checks compare the tensors' shapes with what a call will read or write before anything is
# launched (a short buffer would otherwise be read or written past its end on the GPU).
class ArgumentError(_lib.FoursightError, ValueError):
    """An argument the binding refuses before calling the library: status FS_ERR_INVALID_ARGUMENT,
    as the library reports its own argument errors (and a ValueError)."""

    def __init__(self, who: str, what: str):
        RuntimeError.__init__(self, f"{who}: invalid argument: {what}")
        self.status = _lib.FS_ERR_INVALID_ARGUMENT


def _need(ok: bool, who: str, what: str) -> None:
    if not ok:
        raise ArgumentError(who, what)


def _check_packed(who: str, name: str, pk: Packed, rows: int, K: int, p: int) -> None:
    """pk holds at least `rows` rows of the packed layout: E2M1 codes with a row pitch of K/2
    bytes, the tiled scales of those rows, and (p > 0) bf16 side columns with a pitch of Pp."""
    q = pk.q
    if K > 0:                                       # (a compacted operand of no columns has no codes)
        _need(q.dim() == 2 and q.dtype == torch.uint8 and q.shape[1] * 2 == K and q.stride(1) == 1
              and (q.shape[0] <= 1 or q.stride(0) == K // 2), who,
              f"{name}.q must be uint8 rows of K/2 = {K // 2} bytes")
        _need(q.shape[0] >= rows, who, f"{name} has {q.shape[0]} rows, {rows} are read or written")
        _need(pk.sf.dtype == torch.uint8 and pk.sf.is_contiguous() and pk.sf.numel() >= sf_bytes(rows, K), who,
              f"{name}.sf must hold the {sf_bytes(rows, K)} tiled scale bytes of {rows} rows")
    if p > 0:
        pp, sd = side_cols(p), pk.side
        _need(sd is not None and sd.dim() == 2 and sd.dtype == torch.bfloat16 and sd.shape[0] >= rows
              and sd.shape[1] >= pp and sd.stride(1) == 1 and (sd.shape[0] <= 1 or sd.stride(0) == pp), who,
              f"{name}.side must be bf16 rows of Pp = {pp} columns")


def _check_out(who: str, Y: torch.Tensor, rows: int, cols: int, bf16: bool) -> None:
    _need(Y.dim() == 2 and Y.shape[0] >= rows and Y.shape[1] >= cols and Y.stride(1) == 1, who,
          f"Y must have at least {rows} rows of {cols} columns, unit column stride")
    _need(Y.dtype == (torch.bfloat16 if bf16 else torch.float32), who,
          f"Y must be {'bfloat16' if bf16 else 'float32'} for this plan")


def _check_floats(who: str, name: str, t: torch.Tensor, n: int) -> None:
    _need(t.dtype == torch.float32 and t.numel() >= n, who, f"{name} must hold {n} float32 values")


def _check_gemm_operands(who: str, plan: "Plan", xq: Packed, wq: Packed, alpha, w_rows: int, n_alpha: int) -> None:
    _need(xq.p == wq.p, who, "activations and weights must share p")
    _check_packed(who, "xq", xq, xq.rows, plan.K, xq.p)
    _check_packed(who, "wq", wq, w_rows, plan.K, wq.p)
    _check_floats(who, "alpha", alpha, n_alpha)


def _check_matrix(who: str, name: str, t: torch.Tensor, rows: int, cols: int, dtypes) -> None:
    """t is a 2-D tensor of one of `dtypes` with at least rows x cols and unit column stride (its
    row pitch is passed to the library, which checks it against the width)."""
    _need(t.dim() == 2 and t.dtype in dtypes and t.shape[0] >= rows and t.shape[1] >= cols
          and (t.shape[1] <= 1 or t.stride(1) == 1), who,
          f"{name} must be {'/'.join(str(d) for d in dtypes)} [>= {rows}, >= {cols}] with unit column stride")


def _check_vector(who: str, name: str, t, n: int, dtype) -> None:
    if t is not None:
        _need(t.dtype == dtype and t.is_contiguous() and t.numel() >= n, who, f"{name} must hold {n} {dtype} values")


def fs_channel_stats(X: torch.Tensor, state: StatsState, group: int = 0, row_stride: int = 1, stream=None):
    lib = _lib.load()
    who = "fs_channel_stats"
    _need(0 <= group < state.nprob, who, f"group {group} outside the state's {state.nprob}")
    _need(X.dim() == 2 and X.shape[1] == state.K, who, f"X must be [M, K = {state.K}] (the state's K)")
    _check_matrix(who, "X", X, X.shape[0], state.K, (torch.bfloat16, torch.float32))
    n, s1, s2, amax, flags = state.group(group)
    M, K = X.shape
    check(lib.fs_channel_stats(_ptr(X), _dtype_code(X), M, K, X.stride(0), row_stride, _ptr(n), _ptr(s1),
                               _ptr(s2), _ptr(amax), _ptr(flags), stream_handle(stream)), "fs_channel_stats")


def fs_stats_check(state: StatsState, stream=None):
    check(_lib.load().fs_stats_check(_ptr(state.flags), state.nprob, stream_handle(stream)), "fs_stats_check")


def fs_select_topk(state: StatsState, p: int, opts: int = 0, reset: bool = False, P=None, mask=None, gA=None,
                   stream=None):
    lib = _lib.load()
    dev = state.s1.device
    nprob, K = state.nprob, state.K
    P = torch.empty(nprob, max(p, 1), dtype=torch.int32, device=dev)[:, :p] if P is None else P
    mask = torch.empty(nprob, (K + 31) // 32, dtype=torch.int32, device=dev) if mask is None else mask
    gA = torch.empty(nprob, dtype=torch.float32, device=dev) if gA is None else gA
    who, nw = "fs_select_topk", (K + 31) // 32
    if p > 0:
        _check_matrix(who, "P", P, nprob, p, (torch.int32,))
        _need(nprob <= 1 or P.stride(0) == p, who, f"P rows must be p = {p} apart")
    _check_matrix(who, "mask", mask, nprob, nw, (torch.int32,))
    _need(mask.shape[1] == nw and (nprob <= 1 or mask.stride(0) == nw), who, f"mask rows must be {nw} words")
    _check_vector(who, "gA", gA, nprob, torch.float32)
    check(lib.fs_select_topk(nprob, K, _ptr(state.n), _ptr(state.s1), _ptr(state.s2), _ptr(state.amax),
                             _ptr(state.flags), p, opts, _ptr(P), _ptr(mask), _ptr(gA), int(reset),
                             stream_handle(stream)), "fs_select_topk")
    return P, mask, gA


def compact_cols(K: int, p: int) -> int:
    return _lib.load().fs_compact_cols(K, p)


def _packed_cols(K: int, p: int, opts: int) -> int:
    """Columns of the NVFP4 operand: K, or the compacted width with FS_COMPACT_K."""
    return compact_cols(K, p) if opts & _lib.FS_COMPACT_K else K


def fs_prepare_weights(W: torch.Tensor, mask, p: int, gA: torch.Tensor, opts: int = 0, out: Packed | None = None,
                       gW=None, alpha=None, stream=None):
    lib = _lib.load()
    N, K = W.shape
    out = alloc_packed(N, _packed_cols(K, p, opts), p, W.device) if out is None else out
    gW = torch.empty(1, dtype=torch.float32, device=W.device) if gW is None else gW
    alpha = torch.empty(1, dtype=torch.float32, device=W.device) if alpha is None else alpha
    _check_packed("fs_prepare_weights", "out", out, N, _packed_cols(K, p, opts), p)
    _check_floats("fs_prepare_weights", "gW", gW, 1)
    _check_floats("fs_prepare_weights", "alpha", alpha, 1)
    check(lib.fs_prepare_weights(_ptr(W), _dtype_code(W), N, K, W.stride(0), _ptr(mask) if p else None, p, opts,
                                 _ptr(gA), _ptr(out.q), _ptr(out.sf), _ptr(out.side) if p else None, _ptr(gW),
                                 _ptr(alpha), stream_handle(stream)), "fs_prepare_weights")
    return out, gW, alpha


def fs_quantize_splice(X: torch.Tensor, mask, p: int, gA: torch.Tensor, opts: int = 0, out: Packed | None = None,
                       stream=None):
    lib = _lib.load()
    M, K = X.shape
    out = alloc_packed(M, _packed_cols(K, p, opts), p, X.device) if out is None else out
    _check_packed("fs_quantize_splice", "out", out, M, _packed_cols(K, p, opts), p)
    check(lib.fs_quantize_splice(_ptr(X), _dtype_code(X), M, K, X.stride(0), _ptr(mask) if p else None, p,
                                 _ptr(gA), opts, _ptr(out.q), _ptr(out.sf), _ptr(out.side) if p else None,
                                 stream_handle(stream)), "fs_quantize_splice")
    return out


def fs_quantize_splice_stats(X: torch.Tensor, mask, p: int, gA: torch.Tensor, state: StatsState, group: int = 0,
                             row_stride: int = 1, opts: int = 0, out: Packed | None = None, stream=None):
    """fs_quantize_splice with the CURRENT protected set (mask, p, gA) and fs_channel_stats into
    ``state`` (for the NEXT reselection) in one pass over the bf16 activations X."""
    lib = _lib.load()
    M, K = X.shape
    out = alloc_packed(M, K, p, X.device) if out is None else out
    _check_packed("fs_quantize_splice_stats", "out", out, M, K, p)
    _need(state.K == K, "fs_quantize_splice_stats", f"statistics state of K = {state.K} for K = {K}")
    n, s1, s2, amax, flags = state.group(group)
    check(lib.fs_quantize_splice_stats(_ptr(X), _dtype_code(X), M, K, X.stride(0), _ptr(mask) if p else None, p,
                                       _ptr(gA), opts, _ptr(out.q), _ptr(out.sf), _ptr(out.side) if p else None,
                                       row_stride, _ptr(n), _ptr(s1), _ptr(s2), _ptr(amax), _ptr(flags),
                                       stream_handle(stream)), "fs_quantize_splice_stats")
    return out


def fs_quantize_splice_grouped(X: torch.Tensor, row_offsets: torch.Tensor, masks, p: int, gA: torch.Tensor,
                               opts: int = 0, out: Packed | None = None, max_rows: int | None = None, stream=None):
    lib = _lib.load()
    rows, K = X.shape
    E = row_offsets.numel() - 1
    max_rows = rows if max_rows is None else max_rows
    out = alloc_packed(grouped_rows(max_rows, E), K, p, X.device) if out is None else out
    _check_packed("fs_quantize_splice_grouped", "out", out, grouped_rows(max_rows, E), K, p)
    check(lib.fs_quantize_splice_grouped(_ptr(X), _dtype_code(X), E, _ptr(row_offsets), max_rows, K, X.stride(0),
                                         _ptr(masks) if p else None, p, _ptr(gA), opts, _ptr(out.q), _ptr(out.sf),
                                         _ptr(out.side) if p else None, stream_handle(stream)),
          "fs_quantize_splice_grouped")
    return out


class Plan:
    """Owns an fs_plan (kernel choice for one weight shape plus a device error word)."""

    def __init__(self, N: int, K: int, p_max: int, opts: int = 0):
        self._lib = _lib.load()
        h = C.c_void_p()
        check(self._lib.fs_plan_create(C.byref(h), N, K, p_max, opts), "fs_plan_create")
        self.handle, self.N, self.K, self.p_max, self.opts = h, N, K, p_max, opts

    def check(self, stream=None):
        check(self._lib.fs_plan_check(self.handle, stream_handle(stream)), "fs_plan_check")

    def close(self):
        if self.handle:
            self._lib.fs_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fs_splice_gemm(plan: Plan, xq: Packed, wq: Packed, alpha: torch.Tensor, Y: torch.Tensor | None = None,
                   stream=None):
    lib = _lib.load()
    M = xq.rows
    if Y is None:
        dt = torch.bfloat16 if plan.opts & _lib.FS_OUT_BF16 else torch.float32
        Y = torch.empty(M, plan.N, dtype=dt, device=xq.q.device)
    if M > 0:                                       # an empty batch reads no operand
        _check_gemm_operands("fs_splice_gemm", plan, xq, wq, alpha, plan.N, 1)
        _check_out("fs_splice_gemm", Y, M, plan.N, bool(plan.opts & _lib.FS_OUT_BF16))
    check(lib.fs_splice_gemm(plan.handle, M, xq.p, _ptr(xq.q), _ptr(xq.sf), _ptr(xq.side) if xq.p else None,
                             _ptr(wq.q), _ptr(wq.sf), _ptr(wq.side) if wq.p else None, _ptr(alpha), _ptr(Y),
                             Y.stride(0), stream_handle(stream)), "fs_splice_gemm")
    return Y


def fs_splice_gemm_segmented(plan: Plan, xq: Packed, wq: Packed, alpha: torch.Tensor, seg_start,
                             Y: torch.Tensor | None = None, stream=None):
    """Projections sharing the activations xq, stacked as row ranges seg_start[s]..seg_start[s+1]
    of wq, each with its own alpha[s]; returns Y [M, N] with projection s in those columns."""
    lib = _lib.load()
    M = xq.rows
    seg = [int(v) for v in seg_start]
    arr = (C.c_int32 * len(seg))(*seg)
    if Y is None:
        dt = torch.bfloat16 if plan.opts & _lib.FS_OUT_BF16 else torch.float32
        Y = torch.empty(M, plan.N, dtype=dt, device=xq.q.device)
    if M > 0:
        _check_gemm_operands("fs_splice_gemm_segmented", plan, xq, wq, alpha, plan.N, max(len(seg) - 1, 1))
        _check_out("fs_splice_gemm_segmented", Y, M, plan.N, bool(plan.opts & _lib.FS_OUT_BF16))
    check(lib.fs_splice_gemm_segmented(plan.handle, M, xq.p, _ptr(xq.q), _ptr(xq.sf), _ptr(xq.side) if xq.p else None,
                                       _ptr(wq.q), _ptr(wq.sf), _ptr(wq.side) if wq.p else None, len(seg) - 1, arr,
                                       _ptr(alpha), _ptr(Y), Y.stride(0), stream_handle(stream)),
          "fs_splice_gemm_segmented")
    return Y


def fs_decode_splice_gemm(plan: Plan, X: torch.Tensor, mask, p: int, gA: torch.Tensor, wq: Packed,
                          alpha: torch.Tensor, seg_start=None, xopts: int = 0, Y: torch.Tensor | None = None,
                          stream=None):
    """Decode-path SpliceGEMM (M <= 16) with the activation preparation in the same launch: bf16 X
    [M, K] is masked, quantised and split (as fs_quantize_splice with mask, p, gA, xopts) by the
    GEMM kernel itself.  seg_start as for fs_splice_gemm_segmented (None: one projection)."""
    lib = _lib.load()
    if X.dtype != torch.bfloat16:
        raise TypeError("fs_decode_splice_gemm takes bf16 activations")
    M = X.shape[0]
    if seg_start is None:
        nseg, arr = 1, None
    else:
        seg = [int(v) for v in seg_start]
        nseg, arr = len(seg) - 1, (C.c_int32 * len(seg))(*seg)
    if Y is None:
        dt = torch.bfloat16 if plan.opts & _lib.FS_OUT_BF16 else torch.float32
        Y = torch.empty(M, plan.N, dtype=dt, device=X.device)
    who = "fs_decode_splice_gemm"
    if M > 0:
        _need(X.dim() == 2 and X.shape[1] == plan.K and X.stride(1) == 1, who, f"X must be [M, K = {plan.K}] rows")
        _need(wq.p == p, who, "the weights must be prepared with the same p")
        _check_packed(who, "wq", wq, plan.N, plan.K, p)
        _check_floats(who, "alpha", alpha, nseg)
        _check_floats(who, "gA", gA, 1)
        if p > 0:
            _need(mask is not None and mask.numel() * mask.element_size() >= 4 * ((plan.K + 31) // 32), who,
                  "mask must hold ceil(K/32) words")
        _check_out(who, Y, M, plan.N, bool(plan.opts & _lib.FS_OUT_BF16))
    check(lib.fs_decode_splice_gemm(plan.handle, M, p, _ptr(X), X.stride(0), _ptr(mask) if p else None, _ptr(gA),
                                    xopts, _ptr(wq.q), _ptr(wq.sf), _ptr(wq.side) if wq.p else None, nseg, arr,
                                    _ptr(alpha), _ptr(Y), Y.stride(0), stream_handle(stream)),
          "fs_decode_splice_gemm")
    return Y


def stacked_packed(rows_per_segment, K: int, p: int, device="cuda") -> tuple:
    """One packed weight operand for projections stacked by rows, and per-segment views of it that
    fs_prepare_weights can write (rows of each segment must be a multiple of 128)."""
    total = sum(rows_per_segment)
    pp = side_cols(p)
    q = torch.empty(total, K // 2, dtype=torch.uint8, device=device)
    sf = torch.empty(sf_bytes(total, K), dtype=torch.uint8, device=device)
    side = torch.zeros(total, max(pp, 8), dtype=torch.bfloat16, device=device)[:, :pp]
    views, r0 = [], 0
    for n in rows_per_segment:
        if n % 128:
            raise ValueError("segment rows must be a multiple of 128")
        views.append(Packed(q[r0:r0 + n], sf[sf_bytes(r0, K):sf_bytes(r0 + n, K)], side[r0:r0 + n], n, K, p))
        r0 += n
    return Packed(q, sf, side, total, K, p), views


def fs_splice_gemm_grouped(plan: Plan, row_offsets: torch.Tensor, max_rows: int, xq: Packed, wq: Packed,
                           alpha: torch.Tensor, Y: torch.Tensor | None = None, stream=None):
    lib = _lib.load()
    E = row_offsets.numel() - 1
    if Y is None:
        dt = torch.bfloat16 if plan.opts & _lib.FS_OUT_BF16 else torch.float32
        Y = torch.empty(max_rows, plan.N, dtype=dt, device=xq.q.device)
    who = "fs_splice_gemm_grouped"
    if max_rows > 0:                                # no routed rows: nothing is read or written
        _need(row_offsets.dtype == torch.int64 and E >= 1, who, "row_offsets must be E + 1 int64 values")
        _need(xq.p == wq.p, who, "activations and weights must share p")
        _check_packed(who, "xq", xq, grouped_rows(max_rows, E), plan.K, xq.p)
        _check_packed(who, "wq", wq, E * plan.N, plan.K, wq.p)
        _check_floats(who, "alpha", alpha, E)
        _check_out(who, Y, max_rows, plan.N, bool(plan.opts & _lib.FS_OUT_BF16))
    check(lib.fs_splice_gemm_grouped(plan.handle, E, _ptr(row_offsets), max_rows, xq.p, _ptr(xq.q), _ptr(xq.sf),
                                     _ptr(xq.side) if xq.p else None, _ptr(wq.q), _ptr(wq.sf),
                                     _ptr(wq.side) if wq.p else None, _ptr(alpha), _ptr(Y), Y.stride(0),
                                     stream_handle(stream)), "fs_splice_gemm_grouped")
    return Y


def fs_seq_filter(logp: torch.Tensor, log_tau: float, K1: int, K2: int, lengths=None, G: int = 0, rewards=None,
                  adv=None, stream=None):
    lib = _lib.load()
    S, T = logp.shape
    who = "fs_seq_filter"
    _check_matrix(who, "logp", logp, S, T, (torch.float32,))
    _check_vector(who, "lengths", lengths, S, torch.int32)
    _check_vector(who, "rewards", rewards, S, torch.float32)
    _check_vector(who, "adv", adv, S, torch.float32)
    dev = logp.device
    keep = torch.empty(max(S, 1), dtype=torch.uint8, device=dev)[:S]
    cnt = torch.empty(max(S, 1), dtype=torch.int32, device=dev)[:S]
    run = torch.empty(max(S, 1), dtype=torch.int32, device=dev)[:S]
    if rewards is not None and adv is None:
        adv = torch.empty(S, dtype=torch.float32, device=dev)
    check(lib.fs_seq_filter(_ptr(logp), logp.stride(0), _ptr(lengths), S, T, float(log_tau), K1, K2, G,
                            _ptr(rewards), _ptr(adv), _ptr(keep), _ptr(cnt), _ptr(run), stream_handle(stream)),
          "fs_seq_filter")
    return keep, cnt, run, adv


# ------------------------------------------------------------------------------------------ training side
def _bits16(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.bfloat16:
        raise TypeError("bf16 tensor expected")
    return t


def fs_gemm_bf16(plan: Plan, A: torch.Tensor, B: torch.Tensor, alpha: torch.Tensor | None = None,
                 Y: torch.Tensor | None = None, stream=None):
    """Y [M, N] = alpha * A [M, K] @ B [N, K]^T (bf16 operands, fp32 accumulation)."""
    lib = _lib.load()
    M, K = A.shape
    N = B.shape[0]
    dt = torch.bfloat16 if plan.opts & _lib.FS_OUT_BF16 else torch.float32
    if Y is None:
        Y = torch.empty(M, N, dtype=dt, device=A.device)
    who = "fs_gemm_bf16"
    _check_matrix(who, "A", A, M, K, (torch.bfloat16,))
    _need(B.dim() == 2 and B.shape[1] == K, who, f"B must be [N, K = {K}]")
    _check_matrix(who, "B", B, N, K, (torch.bfloat16,))
    _check_matrix(who, "Y", Y, M, N, (dt,))
    _check_vector(who, "alpha", alpha, 1, torch.float32)
    check(lib.fs_gemm_bf16(plan.handle, M, N, K, _ptr(_bits16(A)), A.stride(0), _ptr(_bits16(B)), B.stride(0),
                           _ptr(alpha), _ptr(Y), Y.stride(0), stream_handle(stream)), "fs_gemm_bf16")
    return Y


def fs_transpose_bf16(src: torch.Tensor, dst: torch.Tensor | None = None, stream=None):
    lib = _lib.load()
    R, C_ = src.shape
    dst = torch.empty(C_, R, dtype=torch.bfloat16, device=src.device) if dst is None else dst
    _check_matrix("fs_transpose_bf16", "src", src, R, C_, (torch.bfloat16,))
    _check_matrix("fs_transpose_bf16", "dst", dst, C_, R, (torch.bfloat16,))
    check(lib.fs_transpose_bf16(R, C_, _ptr(_bits16(src)), src.stride(0), _ptr(dst), dst.stride(0),
                                stream_handle(stream)), "fs_transpose_bf16")
    return dst


def fs_ste_backward(plan: Plan, dY: torch.Tensor, X: torch.Tensor, W: torch.Tensor, work: torch.Tensor | None = None,
                    dX: torch.Tensor | None = None, dW: torch.Tensor | None = None, stream=None):
    """Straight-through backward of the SpliceGEMM forward: (dX, dW) = (dY @ W, dY^T @ X) on bf16 operands."""
    lib = _lib.load()
    M, N = dY.shape
    K = X.shape[1]
    dt = torch.bfloat16 if plan.opts & _lib.FS_OUT_BF16 else torch.float32
    nbytes = lib.fs_ste_backward_work_bytes(M, N, K)
    work = torch.empty(nbytes, dtype=torch.uint8, device=dY.device) if work is None else work
    dX = torch.empty(M, K, dtype=dt, device=dY.device) if dX is None else dX
    dW = torch.empty(N, K, dtype=dt, device=dY.device) if dW is None else dW
    who = "fs_ste_backward"
    _check_matrix(who, "dY", dY, M, N, (torch.bfloat16,))
    _check_matrix(who, "X", X, M, K, (torch.bfloat16,))
    _need(W.dim() == 2 and W.shape[1] == K, who, f"W must be [N, K = {K}]")
    _check_matrix(who, "W", W, N, K, (torch.bfloat16,))
    _check_matrix(who, "dX", dX, M, K, (dt,))
    _check_matrix(who, "dW", dW, N, K, (dt,))
    _check_vector(who, "work", work, nbytes, torch.uint8)
    check(lib.fs_ste_backward(plan.handle, M, N, K, _ptr(_bits16(dY)), dY.stride(0), _ptr(_bits16(X)), X.stride(0),
                              _ptr(_bits16(W)), W.stride(0), _ptr(work), work.numel(), _ptr(dX), dX.stride(0),
                              _ptr(dW), dW.stride(0), stream_handle(stream)), "fs_ste_backward")
    return dX, dW


def fs_grpo_objective(logp: torch.Tensor, logp_old: torch.Tensor, adv: torch.Tensor, eps: float, lengths=None,
                      with_grad: bool = True, stream=None):
    """Eq. 4 with filtered advantages: returns (J [1], seq_obj [S], grad [S, T] or None)."""
    lib = _lib.load()
    S, T = logp.shape
    who = "fs_grpo_objective"
    _check_matrix(who, "logp", logp, S, T, (torch.float32,))
    _check_matrix(who, "logp_old", logp_old, S, T, (torch.float32,))
    _need(S <= 1 or logp_old.stride(0) == logp.stride(0), who, "logp and logp_old must share their row pitch")
    _check_vector(who, "adv", adv, S, torch.float32)
    _check_vector(who, "lengths", lengths, S, torch.int32)
    seq = torch.empty(max(S, 1), dtype=torch.float32, device=logp.device)[:S]
    J = torch.empty(1, dtype=torch.float32, device=logp.device)
    grad = torch.empty(S, T, dtype=torch.float32, device=logp.device) if with_grad else None
    check(lib.fs_grpo_objective(_ptr(logp), _ptr(logp_old), logp.stride(0), _ptr(lengths), S, T, _ptr(adv),
                                float(eps), _ptr(seq), _ptr(J), _ptr(grad), grad.stride(0) if grad is not None else T,
                                stream_handle(stream)), "fs_grpo_objective")
    return J, seq, grad


def fs_k3_kl(logp_train: torch.Tensor, logp_roll: torch.Tensor, lengths=None, stream=None):
    """K3 estimates of KL(pi_rollout || pi_train): (per-sequence means [S], batch mean [1])."""
    lib = _lib.load()
    S, T = logp_train.shape
    who = "fs_k3_kl"
    _check_matrix(who, "logp_train", logp_train, S, T, (torch.float32,))
    _check_matrix(who, "logp_roll", logp_roll, S, T, (torch.float32,))
    _need(S <= 1 or logp_roll.stride(0) == logp_train.stride(0), who, "both log-prob arrays must share their row pitch")
    _check_vector(who, "lengths", lengths, S, torch.int32)
    seq = torch.empty(max(S, 1), dtype=torch.float32, device=logp_train.device)[:S]
    batch = torch.empty(1, dtype=torch.float32, device=logp_train.device)
    work = torch.empty(max(lib.fs_k3_work_bytes(S), 8), dtype=torch.uint8, device=logp_train.device)
    check(lib.fs_k3_kl(_ptr(logp_train), _ptr(logp_roll), logp_train.stride(0), _ptr(lengths), S, T, _ptr(seq),
                       _ptr(batch), _ptr(work), stream_handle(stream)), "fs_k3_kl")
    return seq, batch
