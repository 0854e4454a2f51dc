"""Muon optimizer step for sets of 2D weight matrices on B200 (sm_100a).

A thin Python binding over the C ABI in ``include/muon_ns.h``: it only turns
torch tensors into device pointers, shape tables and the current CUDA
stream. Every stage of the step runs in the library's CUDA kernels; there is
no Python or CPU fallback.

    import torch, muon_newton_schulz_03_b200 as muon
    opt = muon.Muon(device=0)                     # Moonlight scale, bf16 NS
    opt.step(params, grads, momenta, lr=2e-4)     # lists of 2D CUDA tensors

Readings of the method (see the C header): momentum EMA with the Nesterov
blend, u / (||u||_F + 1e-7), five quintic Newton-Schulz steps with
(3.4445, -4.7750, 2.0315) on the short side, scale * lr update with decoupled
weight decay ("About Muon: Why Not Adam", "The whole thing, in about forty
lines").
"""

from __future__ import annotations

import ctypes

from ._lib import EXPORTED, MuonConfig, MuonError, check, lib_path, load

__all__ = ["Muon", "MuonError", "plan_query", "x_layout", "round_up", "split_rows", "SCALE_MODES",
           "DEFAULT_COEFFS", "EXPORTED", "lib_path", "load"]

DEFAULT_COEFFS = (3.4445, -4.7750, 2.0315)
SCALE_MODES = {"moonlight": 0, "jordan": 1, "bernstein": 2, "none": 3}
PRECISIONS = {"bf16": 0, "fp32": 1}
ALGORITHMS = {"standard": 0, "gram": 1}
FLAG_GRAD_BF16 = 1


def round_up(x: int, k: int) -> int:
    return (x + k - 1) // k * k


def _ptr_array(ptrs):
    arr = (ctypes.c_void_p * len(ptrs))()
    for i, p in enumerate(ptrs):
        arr[i] = p
    return arr


def _shapes_array(shapes):
    arr = (ctypes.c_int32 * (3 * len(shapes)))()
    for i, (m, n, f) in enumerate(shapes):
        arr[3 * i], arr[3 * i + 1], arr[3 * i + 2] = m, n, f
    return arr


def _coeffs(coeffs):
    if coeffs is None:
        return None
    c = (ctypes.c_float * 3)(*[float(v) for v in coeffs])
    return c


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check_2d(t, what, dtypes, device=None, contiguous=True):
    import torch
    if t.dim() != 2:
        raise ValueError(f"{what} must be 2D (Muon applies to 2D weight matrices), got shape {tuple(t.shape)}")
    if t.dtype not in dtypes:
        raise TypeError(f"{what} must have dtype in {dtypes}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{what} must be on {device}, got {t.device}")
    return torch


def _bad_matrix(i, p, g, m, host):
    """Raise the precise error for matrix i of a step's lists."""
    import torch
    dev = None if host else p.device
    _check_2d(p, f"params[{i}]", (torch.float32,), dev)
    _check_2d(m, f"momenta[{i}]", (torch.float32,), dev)
    if m.shape != p.shape:
        raise ValueError(f"momenta[{i}] shape {tuple(m.shape)} != params shape {tuple(p.shape)}")
    if g is not None:
        _check_2d(g, f"grads[{i}]", (torch.float32, torch.bfloat16), dev)
        if g.shape != p.shape:
            raise ValueError(f"grads[{i}] shape {tuple(g.shape)} != params shape {tuple(p.shape)}")
    for t, what in ((p, "params"), (m, "momenta"), (g, "grads")):
        if t is not None and (t.device.type == "cpu") != host:
            where = "in host memory" if host else "on a CUDA device"
            raise ValueError(f"{what}[{i}] must be {where}")
    raise ValueError(f"matrix {i}: invalid tensors")   # not reached


def _marshal_step(params, grads, momenta, host=False, device_index=None):
    """Pointer arrays and shape table of a step's matrix lists.

    Every tensor is 2D and contiguous; params and momenta are fp32, grads
    fp32 or bf16 (None skips the matrix); the tensors of one matrix have one
    shape and one device, which is host memory for ``host`` and a CUDA device
    otherwise (the C side cannot see tensor sizes, so they are checked
    here; with ``device_index`` the device must be that CUDA device). Returns
    (params, grads, momenta, shapes, count) as ctypes arrays.
    """
    import torch
    f32, bf16 = torch.float32, torch.bfloat16
    pp, gp, mp, flat = [], [], [], []
    for i, (p, g, m) in enumerate(zip(params, grads, momenta, strict=True)):
        dev = p.device
        ok = (p.dim() == 2 and p.dtype == f32 and p.is_contiguous() and (dev.type == "cpu") == host
              and m.dtype == f32 and m.is_contiguous() and m.shape == p.shape and m.device == dev)
        if ok and g is not None:
            ok = (g.dtype == f32 or g.dtype == bf16) and g.is_contiguous() and g.shape == p.shape and g.device == dev
        if not ok:
            _bad_matrix(i, p, g, m, host)
        if device_index is not None and not host and dev.index != device_index:
            raise ValueError(f"params[{i}] is on {dev}, the handle on cuda:{device_index}")
        pp.append(p.data_ptr())
        mp.append(m.data_ptr())
        if g is None:
            gp.append(None)
            flat += (p.shape[0], p.shape[1], 0)
        else:
            gp.append(g.data_ptr())
            flat += (p.shape[0], p.shape[1], FLAG_GRAD_BF16 if g.dtype == bf16 else 0)
    n = len(pp)
    return ((ctypes.c_void_p * n)(*pp), (ctypes.c_void_p * n)(*gp), (ctypes.c_void_p * n)(*mp),
            (ctypes.c_int32 * (3 * n))(*flat), n)


def x_layout(m: int, n: int, dtype, device):
    """An empty X-layout buffer: row-major m x round_up(n, 8)."""
    import torch
    return torch.empty((m, round_up(n, 8)), dtype=dtype, device=device)


def _blocks(rows, spec):
    if spec is None:
        return [rows]
    if isinstance(spec, int):
        if spec < 1 or rows % spec:
            raise ValueError(f"row split {spec} does not divide {rows} rows")
        return [spec] * (rows // spec)
    spec = [int(h) for h in spec]
    if sum(spec) != rows or min(spec) < 1:
        raise ValueError(f"row blocks {spec} do not sum to {rows} rows")
    return spec


def split_rows(params, grads, momenta, row_splits):
    """Row-block views for split Muon (see Muon.step)."""
    if len(row_splits) != len(params):
        raise ValueError("row_splits needs one entry per matrix")
    P, G, M = [], [], []
    for p, g, m, spec in zip(params, grads, momenta, row_splits):
        r0 = 0
        for h in _blocks(p.shape[0], spec):
            P.append(p[r0:r0 + h])
            G.append(None if g is None else g[r0:r0 + h])
            M.append(m[r0:r0 + h])
            r0 += h
    return P, G, M


def plan_query(shapes, ns_precision: str = "bf16", small_path: bool = True, cta_pair: bool = False):
    """Integer plan tables of a shape table (list of (m, n) or (m, n, flags)).

    Returns dict(ws_bytes, region_offsets [count][4], tiles (gram, poly,
    comb lists of (mat, ti, tj)), small (list of small-path matrices),
    chunk_prefix). Needs no GPU.
    """
    lib = load()
    sh = [(int(s[0]), int(s[1]), int(s[2]) if len(s) > 2 else 0) for s in shapes]
    count = len(sh)
    arr = _shapes_array(sh)
    prec = PRECISIONS[ns_precision]
    sp = (1 if small_path else 0) | (2 if cta_pair else 0)
    nt = (ctypes.c_int32 * 4)()
    ws = ctypes.c_int64()
    check(lib.muon_plan_query(arr, count, prec, sp, ctypes.byref(ws), None, nt, None, None))
    total = nt[0] + nt[1] + nt[2] + nt[3]
    offs = (ctypes.c_int64 * (4 * count))()
    tiles = (ctypes.c_int32 * (3 * max(total, 1)))()
    pref = (ctypes.c_int64 * (count + 1))()
    check(lib.muon_plan_query(arr, count, prec, sp, ctypes.byref(ws), offs, nt, tiles, pref))
    tl = [(tiles[3 * k], tiles[3 * k + 1], tiles[3 * k + 2]) for k in range(total)]
    a, b, c = nt[0], nt[0] + nt[1], nt[0] + nt[1] + nt[2]
    return {
        "ws_bytes": ws.value,
        "region_offsets": [list(offs[4 * i:4 * i + 4]) for i in range(count)],
        "tiles": (tl[:a], tl[a:b], tl[b:c]),
        "small": [t[0] for t in tl[c:]],
        "chunk_prefix": list(pref),
    }


def plan_groups(shapes, cap_bytes: int, ns_precision: str = "bf16", small_path: bool = True,
                cta_pair: bool = False):
    """Matrix groups under a workspace cap. Returns dict(bounds (group g is
    matrices bounds[g]..bounds[g+1]-1), region_offsets [count][4],
    ws_bytes). Needs no GPU."""
    lib = load()
    sh = [(int(s[0]), int(s[1]), int(s[2]) if len(s) > 2 else 0) for s in shapes]
    count = len(sh)
    arr = _shapes_array(sh)
    sp = (1 if small_path else 0) | (2 if cta_pair else 0)
    ng = ctypes.c_int32()
    bounds = (ctypes.c_int32 * (count + 1))()
    offs = (ctypes.c_int64 * (4 * count))()
    ws = ctypes.c_int64()
    check(lib.muon_plan_groups(arr, count, PRECISIONS[ns_precision], sp, int(cap_bytes), ctypes.byref(ng), bounds,
                               offs, ctypes.byref(ws)))
    return {"bounds": list(bounds[:ng.value + 1]), "region_offsets": [list(offs[4 * i:4 * i + 4]) for i in range(count)],
            "ws_bytes": ws.value}


class Muon:
    """A handle of the Muon library on one CUDA device."""

    def __init__(self, device: int = 0, scale_mode: str = "moonlight", extra_scale: float = 1.0,
                 ns_precision: str = "bf16", check_nonfinite: bool = False, num_sms: int = 0,
                 workspace_cap_bytes: int = 0, wait_timeout_s: float = 2.0, small_path: bool = True,
                 cta_pair: bool = False, ns_algorithm: str = "standard", deterministic: bool = False,
                 fused_apply: bool = True):
        self._lib = load()
        cfg = MuonConfig()
        check(self._lib.muon_config_init(ctypes.byref(cfg)))
        cfg.scale_mode = SCALE_MODES[scale_mode]
        cfg.extra_scale = float(extra_scale)
        cfg.ns_precision = PRECISIONS[ns_precision]
        cfg.check_nonfinite = int(bool(check_nonfinite))
        cfg.num_sms = int(num_sms)
        cfg.workspace_cap_bytes = int(workspace_cap_bytes)
        cfg.wait_timeout_s = float(wait_timeout_s)
        cfg.small_path = int(bool(small_path))
        cfg.cta_pair = int(bool(cta_pair))
        cfg.ns_algorithm = ALGORITHMS[ns_algorithm]
        cfg.deterministic = int(bool(deterministic))
        cfg.fused_apply = int(bool(fused_apply))
        h = ctypes.c_void_p()
        check(self._lib.muon_init(int(device), ctypes.byref(cfg), ctypes.byref(h)))
        self._h = h
        self.device = device
        self.ns_precision = ns_precision
        self.small_path = bool(small_path)
        self.cta_pair = bool(cta_pair)
        self.ns_algorithm = ns_algorithm
        # True when this handle's steps may write p' in their last combine and
        # store no O (muon_config.fused_apply); a step does so when no active
        # matrix is on the small path and every row is 16-byte aligned.
        self.fused_apply = (bool(fused_apply) and ns_precision == "bf16" and ns_algorithm == "standard"
                            and not cta_pair)

    # -- lifetime -----------------------------------------------------------
    def close(self):
        if getattr(self, "_h", None):
            self._lib.muon_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def _xdtype(self):
        import torch
        return torch.float32 if self.ns_precision == "fp32" else torch.bfloat16

    # -- full step ----------------------------------------------------------
    def step(self, params, grads, momenta, lr, beta=0.95, nesterov=True, wd=0.1, ns_steps=5, coeffs=None,
             stream=None, row_splits=None):
        """One Muon step, in place on params and momenta (lists of CUDA tensors).

        A ``None`` gradient skips its matrix. ``row_splits`` (optional, one
        entry per matrix) requests split Muon: ``None`` keeps the matrix whole,
        an int h cuts it into row blocks of h rows, a list gives the block
        heights; every block is then a Muon matrix of its own (its rows are
        contiguous, so the blocks are passed as views, no copy).
        """
        if row_splits is not None:
            params, grads, momenta = split_rows(params, grads, momenta, row_splits)
        pa, ga, ma, sa, n = _marshal_step(params, grads, momenta, device_index=self.device)
        check(self._lib.muon_step(self._h, pa, ga, ma, sa, n, float(lr), float(beta), int(bool(nesterov)),
                                  float(wd), int(ns_steps), _coeffs(coeffs), _stream_handle(stream)))

    def step_schedule(self, params, grads, momenta, coeff_table, lr, beta=0.95, nesterov=True, wd=0.1,
                      stream=None):
        """One Muon step whose Newton-Schulz iteration t uses coeff_table[t] = (a, b, c)."""
        import torch
        rows = [tuple(float(v) for v in r) for r in coeff_table]
        if not rows or any(len(r) != 3 for r in rows):
            raise ValueError("coeff_table must be a non-empty list of (a, b, c)")
        table = (ctypes.c_float * (3 * len(rows)))(*[v for r in rows for v in r])
        pa, ga, ma, sa, n = _marshal_step(params, grads, momenta, device_index=self.device)
        check(self._lib.muon_step_schedule(self._h, pa, ga, ma, sa, n, float(lr), float(beta), int(bool(nesterov)),
                                           float(wd), len(rows), table, len(rows), _stream_handle(stream)))

    def qk_clip(self, weights, s_max, head_rows, tau=100.0, stream=None):
        """QK-Clip in place on W_q / W_k weights (fp32 CUDA tensors).

        s_max: one float32 CUDA tensor per weight with the largest attention
        logit of each head; head_rows: rows per head (int or one per weight).
        """
        import torch
        if isinstance(head_rows, int):
            head_rows = [head_rows] * len(weights)
        shapes = []
        for i, (w, s, hr) in enumerate(zip(weights, s_max, head_rows, strict=True)):
            _check_2d(w, f"weights[{i}]", (torch.float32,))
            if s.dtype != torch.float32 or not s.is_contiguous() or s.numel() * hr != w.shape[0]:
                raise ValueError(f"s_max[{i}] must be a contiguous float32 tensor with one entry per head")
            shapes.append((w.shape[0], w.shape[1], int(hr)))
        check(self._lib.muon_qk_clip(self._h, _ptr_array([w.data_ptr() for w in weights]), _shapes_array(shapes),
                                     _ptr_array([s.data_ptr() for s in s_max]), len(weights), float(tau),
                                     _stream_handle(stream)))

    def step_host(self, params, grads, momenta, lr, beta=0.95, nesterov=True, wd=0.1, ns_steps=5,
                  coeffs=None, stream=None):
        """The same step with every tensor in host memory (pinned for async copies).

        The copies and the kernels are enqueued on ``stream``; synchronise it
        before reading params / momenta.
        """
        pa, ga, ma, sa, n = _marshal_step(params, grads, momenta, host=True)
        check(self._lib.muon_step_host(self._h, pa, ga, ma, sa, n, float(lr), float(beta), int(bool(nesterov)),
                                       float(wd), int(ns_steps), _coeffs(coeffs), _stream_handle(stream)))

    # -- stages -------------------------------------------------------------
    def momentum_norm(self, grads, momenta, ys, sumsq, beta=0.95, nesterov=True, stream=None):
        """Stage 1: momentum in place, y = cast(u) in X layout, sumsq[i] = sum u^2."""
        import torch
        shapes = []
        for i, (g, m, y) in enumerate(zip(grads, momenta, ys, strict=True)):
            _check_2d(m, f"momenta[{i}]", (torch.float32,))
            if g is not None:
                _check_2d(g, f"grads[{i}]", (torch.float32, torch.bfloat16), m.device)
                if g.shape != m.shape:
                    raise ValueError(f"grads[{i}] shape {tuple(g.shape)} != momenta shape {tuple(m.shape)}")
            self._check_on_device(m, f"momenta[{i}]")
            self._check_x(y, m.shape, f"y[{i}]")
            shapes.append((m.shape[0], m.shape[1],
                           FLAG_GRAD_BF16 if (g is not None and g.dtype == torch.bfloat16) else 0))
        self._check_sumsq(sumsq, len(shapes))
        check(self._lib.muon_momentum_norm(self._h, _ptr_array([_ptr(g) for g in grads]),
                                           _ptr_array([m.data_ptr() for m in momenta]),
                                           _ptr_array([y.data_ptr() for y in ys]), sumsq.data_ptr(),
                                           _shapes_array(shapes), len(shapes), float(beta), int(bool(nesterov)),
                                           _stream_handle(stream)))

    def newton_schulz(self, x_in, x_out, shapes, sumsq=None, ns_steps=5, coeffs=None, stream=None):
        """Stage 2 on X-layout buffers; shapes is a list of (m, n)."""
        sh = [(int(m), int(n), 0) for (m, n) in shapes]
        for i, ((m, n, _), xi, xo) in enumerate(zip(sh, x_in, x_out, strict=True)):
            self._check_x(xi, (m, n), f"x_in[{i}]")
            self._check_x(xo, (m, n), f"x_out[{i}]")
        if sumsq is not None:
            self._check_sumsq(sumsq, len(sh))
        check(self._lib.muon_newton_schulz(self._h, _ptr_array([x.data_ptr() for x in x_in]),
                                           _ptr_array([x.data_ptr() for x in x_out]),
                                           None if sumsq is None else sumsq.data_ptr(), _shapes_array(sh),
                                           len(sh), int(ns_steps), _coeffs(coeffs), _stream_handle(stream)))

    def apply(self, params, os_, lr, wd, sumsq=None, stream=None):
        """Stage 3: params <- params (1 - lr wd) - lr scale o_scale O."""
        import torch
        shapes = []
        for i, (p, o) in enumerate(zip(params, os_, strict=True)):
            _check_2d(p, f"params[{i}]", (torch.float32,))
            self._check_on_device(p, f"params[{i}]")
            if o is not None:
                self._check_x(o, p.shape, f"o[{i}]")
            shapes.append((p.shape[0], p.shape[1], 0))
        if sumsq is not None:
            self._check_sumsq(sumsq, len(shapes))
        check(self._lib.muon_apply(self._h, _ptr_array([p.data_ptr() for p in params]),
                                   _ptr_array([_ptr(o) for o in os_]),
                                   None if sumsq is None else sumsq.data_ptr(), _shapes_array(shapes),
                                   len(shapes), float(lr), float(wd), _stream_handle(stream)))

    def _check_on_device(self, t, what):
        if t.device.type != "cuda" or t.device.index != self.device:
            raise ValueError(f"{what} must be on cuda:{self.device}, got {t.device}")

    def _check_sumsq(self, sumsq, count):
        import torch
        if sumsq.dtype != torch.float64 or sumsq.numel() < count or not sumsq.is_contiguous():
            raise ValueError("sumsq must be a contiguous float64 tensor with one entry per matrix")
        self._check_on_device(sumsq, "sumsq")

    def _check_x(self, x, shape, what):
        self._check_on_device(x, what)
        m, n = int(shape[0]), int(shape[1])
        if x.dtype != self._xdtype():
            raise TypeError(f"{what} must be {self._xdtype()} in {self.ns_precision} mode")
        if tuple(x.shape) != (m, round_up(n, 8)) or not x.is_contiguous():
            raise ValueError(f"{what} must be a contiguous X-layout buffer of shape ({m}, {round_up(n, 8)})")

    # -- inspection ---------------------------------------------------------
    def status(self, stream=None):
        """(code, error_word, nonfinite_count); waits for the stream."""
        ew = ctypes.c_int32()
        nf = ctypes.c_uint64()
        code = self._lib.muon_get_status(self._h, _stream_handle(stream), ctypes.byref(ew), ctypes.byref(nf))
        return code, ew.value, nf.value

    def workspace(self):
        base = ctypes.c_void_p()
        size = ctypes.c_size_t()
        check(self._lib.muon_workspace_ptr(self._h, ctypes.byref(base), ctypes.byref(size)))
        return base.value or 0, size.value

    KERNEL_KINDS = ("momentum_norm", "ns_gram", "ns_poly", "ns_comb", "apply", "scale_copy", "ns_fp32", "ns_small",
                    "norm_reduce", "ns_sym")

    def profile_enable(self, max_calls: int):
        """Record CUDA events around every kernel of the next max_calls calls."""
        check(self._lib.muon_profile_enable(self._h, int(max_calls)))

    def profile_read(self, max_entries: int = 65536):
        """[(kind, ms)] of the recorded kernels, in launch order; clears the record."""
        kinds = (ctypes.c_int32 * max_entries)()
        ms = (ctypes.c_float * max_entries)()
        n = ctypes.c_int32()
        check(self._lib.muon_profile_read(self._h, kinds, ms, max_entries, ctypes.byref(n)))
        return [(self.KERNEL_KINDS[kinds[i]], ms[i]) for i in range(n.value)]

    def last_launch_count(self) -> int:
        n = ctypes.c_int32()
        check(self._lib.muon_last_launch_count(self._h, ctypes.byref(n)))
        return n.value
