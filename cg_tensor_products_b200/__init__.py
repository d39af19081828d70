"""Python binding of libetp.so, the B200 edge-wise equivariant tensor product library.

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels (see include/etp.h for the operation, layouts and conventions).
PyTorch supplies device memory and the current stream. There is no CPU path:
tensors must live on a CUDA device, and a missing library raises.

    plan = Plan("0..3", 3, "0..3", C=128)
    out = forward(plan, row_ptr, src, r, x, w)
    rev_ptr, rev_perm, dst = build_reverse_csr(N, row_ptr, src)
    gx, gw, gr = backward(plan, row_ptr, src, rev_ptr, rev_perm, dst, r, x, w, grad_out)
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libetp.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "etp.h")

ETP_OK, ETP_ERR_INVALID_ARG, ETP_ERR_UNSUPPORTED, ETP_ERR_BAD_CSR = 0, 1, 2, 3
ETP_ERR_CUDA, ETP_ERR_ALLOC, ETP_ERR_WORKSPACE, ETP_ERR_TOO_LARGE = 4, 5, 6, 7
STATIC_MAX_NODES = STATIC_MAX_EDGES = 1 << 18
FRAME_FLOATS = 88  # floats of one edge frame record (ETP_FRAME_FLOATS)
ETP_F32 = 0
CSR_BAD_ENDPOINTS, CSR_NOT_MONOTONE, CSR_SRC_RANGE = 1, 2, 4

_lib = None


class EtpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _load().etp_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{where}: {msg} (status {status})")


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m cg_tensor_products_b200.build` "
                           "(or __graft_entry__.build()); there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "etp_plan_create": [ctypes.POINTER(vp), ctypes.c_char_p, i32, ctypes.c_char_p, i32, i32],
        "etp_plan_info": [vp, vp, vp, vp, vp, vp],
        "etp_plan_couplings": [vp, vp, vp, vp, vp, vp, vp],
        "etp_plan_destroy": [vp],
        "etp_plan_frames_advised": [vp, i32, ctypes.POINTER(i32)],
        "etp_edge_frames": [vp, i32, vp, vp, vp],
        "etp_tp_workspace_size": [vp, i32, i32, i32, ctypes.POINTER(sz)],
        "etp_forward": [vp, i32, i32] + [vp] * 7 + [vp, sz, vp],
        "etp_backward": [vp, i32, i32] + [vp] * 13 + [vp, sz, vp],
        "etp_double_backward": [vp, i32, i32] + [vp] * 16 + [vp, sz, vp],
        "etp_cart_forward": [vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "etp_cart_backward": [vp, i32, i32] + [vp] * 12 + [vp, sz, vp],
        "etp_assemble_forces": [i32, i32, vp, vp, vp, vp, vp, vp, vp, vp],
        "etp_node_product": [vp, i32, i32, i32, vp, vp, vp, vp],
        "etp_node_product_ops": [vp, i32, ctypes.POINTER(i32)],
        "etp_radial_workspace_size": [vp, i32, i32, i32, ctypes.POINTER(sz)],
        "etp_radial_forward": [vp, i32, i32, i32, ctypes.c_float, vp, vp, vp, vp, vp, sz, vp],
        "etp_radial_backward": [vp, i32, i32, i32, ctypes.c_float, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "etp_fused_workspace_size": [vp, i32, i32, i32, ctypes.POINTER(sz)],
        "etp_fused_forward": [vp, i32, i32, vp, vp, vp, vp, i32, i32, ctypes.c_float, vp, vp, vp, vp, sz, vp],
        "etp_reverse_csr_workspace_size": [i32, i32, ctypes.POINTER(sz)],
        "etp_build_reverse_csr": [i32, i32, vp, vp, vp, vp, vp, vp, sz, vp],
        "etp_build_reverse_csr_static": [i32, i32, vp, vp, vp, vp, vp, vp],
        "etp_validate_csr": [i32, i32, vp, vp, vp, vp],
        "etp_locality_schedule_workspace_size": [i32, i32, ctypes.POINTER(sz)],
        "etp_build_locality_schedule": [i32, i32, vp, vp, vp, ctypes.c_float, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "etp_forward_ordered": [vp, i32, i32] + [vp] * 10 + [sz, vp],
        "etp_backward_ordered": [vp, i32, i32] + [vp] * 13 + [sz, vp],
        "etp_device_fault": [vp],
        "etp_status_string": [i32],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "etp_status_string" else ctypes.c_int
    _lib = lib
    return lib


def declared_symbols() -> list:
    """Function names declared in include/etp.h."""
    with open(HEADER_PATH) as f:
        txt = f.read()
    return re.findall(r"ETP_API\s+[\w\s\*]+?\b(etp_\w+)\s*\(", txt)


def _check(status: int, where: str):
    if status != ETP_OK:
        raise EtpError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(*ts):
    """The one CUDA device all given tensors live on (None entries are skipped)."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors: this library has no CPU path")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on different devices ({dev}, {t.device})")
    return dev


def _launch(dev, where: str, fn, *args, stream=None):
    """Call library function `fn(*args, stream)` with the tensors' device current.

    The library launches on the current device and on the stream it is given, so
    both must be the tensors' device: torch's current stream of `dev`, or a
    caller's stream, which must belong to `dev`."""
    import torch

    s = stream if stream is not None else torch.cuda.current_stream(dev)
    if s.device != dev:
        raise ValueError(f"{where}: stream on {s.device}, tensors on {dev}")
    with torch.cuda.device(dev):
        _check(fn(*args, ctypes.c_void_p(s.cuda_stream)), where)


def _expect(t, name: str, dtype: str, shape: tuple):
    """Raise ValueError unless t (if given) has the dtype ('float32' / 'int32' / 'uint8') and the
    shape (None entries match any size); checked before anything is launched."""
    if t is None:
        return
    if str(t.dtype) != "torch." + dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.dim() != len(shape) or any(want is not None and got != want for got, want in zip(t.shape, shape)):
        raise ValueError(f"{name}: expected shape {tuple('*' if v is None else v for v in shape)}, "
                         f"got {tuple(t.shape)}")


def _check_graph(row_ptr, src, N: int, E: int):
    _expect(row_ptr, "row_ptr", "int32", (N + 1,))
    _expect(src, "src", "int32", (E,))


class Plan:
    """A tensor-product plan: irreps in x harmonics 0..sh_lmax -> irreps out, C channels, fp32."""

    def __init__(self, irreps_in: str, sh_lmax: int, irreps_out: str, C: int):
        lib = _load()
        h = ctypes.c_void_p()
        _check(lib.etp_plan_create(ctypes.byref(h), irreps_in.encode(), int(sh_lmax), irreps_out.encode(),
                                   int(C), ETP_F32), "etp_plan_create")
        self._h = h
        self.C = int(C)
        n_paths, d_in, d_sh, d_out = (ctypes.c_int() for _ in range(4))
        _check(lib.etp_plan_info(h, ctypes.byref(n_paths), ctypes.byref(d_in), ctypes.byref(d_sh),
                                 ctypes.byref(d_out), None), "etp_plan_info")
        self.n_paths, self.dim_in, self.dim_sh, self.dim_out = n_paths.value, d_in.value, d_sh.value, d_out.value
        arr = (ctypes.c_int * (3 * self.n_paths))()
        _check(lib.etp_plan_info(h, None, None, None, None, arr), "etp_plan_info")
        self.paths = [tuple(arr[3 * p:3 * p + 3]) for p in range(self.n_paths)]

    @property
    def handle(self):
        return self._h

    def couplings(self):
        """(path_off, m1, m2, m3, val) of the coefficients compiled into the kernels."""
        lib = _load()
        nnz = ctypes.c_int()
        _check(lib.etp_plan_couplings(self._h, ctypes.byref(nnz), None, None, None, None, None), "couplings")
        n = nnz.value
        off = (ctypes.c_int * (self.n_paths + 1))()
        m1, m2, m3 = ((ctypes.c_int * n)() for _ in range(3))
        val = (ctypes.c_double * n)()
        _check(lib.etp_plan_couplings(self._h, ctypes.byref(nnz), off, m1, m2, m3, val), "couplings")
        return list(off), list(m1), list(m2), list(m3), list(val)

    def frames_advised(self, E: int) -> bool:
        """Whether precomputed edge frame records pay for E edges (etp_plan_frames_advised)."""
        v = ctypes.c_int()
        _check(_load().etp_plan_frames_advised(self._h, int(E), ctypes.byref(v)), "etp_plan_frames_advised")
        return bool(v.value)

    def close(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.etp_plan_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def edge_frames(plan: Plan, r, frames=None, stream=None):
    """Per-edge frame records [E][FRAME_FLOATS] for r (launches etp_edge_frames)."""
    import torch

    _expect(r, "r", "float32", (None, 3))
    E = r.shape[0]
    if frames is None:
        frames = torch.empty((E, FRAME_FLOATS), device=r.device, dtype=torch.float32)
    _expect(frames, "frames", "float32", (E, FRAME_FLOATS))
    dev = _need_cuda(r, frames)
    _launch(dev, "etp_edge_frames", _load().etp_edge_frames, plan.handle, E, _ptr(r), _ptr(frames), stream=stream)
    return frames


def tp_workspace_size(plan: Plan, N: int, E: int, ordered: bool = False, device=None) -> int:
    """Bytes of partial-row workspace forward/backward (ordered: their schedule variants) need
    (etp_tp_workspace_size, answered for `device`, default the current one)."""
    import torch

    b = ctypes.c_size_t()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        _check(_load().etp_tp_workspace_size(plan.handle, int(N), int(E), int(bool(ordered)), ctypes.byref(b)),
               "tp_workspace_size")
    return b.value


def _tp_workspace(plan, N, E, ordered, workspace, dev):
    """The caller's workspace (checked), or a new one of the needed size on dev."""
    import torch

    if workspace is None:
        n = tp_workspace_size(plan, N, E, ordered, dev)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    _expect(workspace, "workspace", "uint8", (None,))
    return workspace


def forward(plan: Plan, row_ptr, src, r, x, w, out=None, frames=None, workspace=None, stream=None):
    """out[i] = sum over row i of the weighted tensor products (launches etp_forward).
    frames: None, or edge_frames(plan, r) (then the kernel reads those instead of building them).
    workspace: uint8 device tensor of tp_workspace_size bytes (allocated when None)."""
    import torch

    N, E = row_ptr.numel() - 1, src.numel()
    _check_graph(row_ptr, src, N, E)
    _expect(r, "r", "float32", (E, 3))
    _expect(frames, "frames", "float32", (E, FRAME_FLOATS))
    _expect(x, "x", "float32", (N, plan.dim_in, plan.C))
    _expect(w, "w", "float32", (E, plan.n_paths, plan.C))
    if out is None:
        out = torch.empty((N, plan.dim_out, plan.C), device=x.device, dtype=torch.float32)
    _expect(out, "out", "float32", (N, plan.dim_out, plan.C))
    dev = _need_cuda(row_ptr, src, r, frames, x, w, out)
    workspace = _tp_workspace(plan, N, E, False, workspace, dev)
    _need_cuda(out, workspace)
    _launch(dev, "etp_forward", _load().etp_forward, plan.handle, N, E, _ptr(row_ptr), _ptr(src), _ptr(r),
            _ptr(frames), _ptr(x), _ptr(w), _ptr(out), _ptr(workspace), workspace.numel(), stream=stream)
    return out


def backward(plan: Plan, row_ptr, src, rev_ptr, rev_perm, dst, r, x, w, grad_out,
             want=("x", "w", "r"), grad_x=None, grad_w=None, grad_r=None, frames=None, workspace=None, stream=None):
    """(grad_x, grad_w, grad_r) for the cotangent grad_out (launches etp_backward); unwanted ones are None."""
    import torch

    N, E = row_ptr.numel() - 1, src.numel()
    _check_graph(row_ptr, src, N, E)
    _expect(rev_ptr, "rev_ptr", "int32", (N + 1,))
    _expect(rev_perm, "rev_perm", "int32", (E,))
    _expect(dst, "dst", "int32", (E,))
    _expect(r, "r", "float32", (E, 3))
    _expect(frames, "frames", "float32", (E, FRAME_FLOATS))
    _expect(x, "x", "float32", (N, plan.dim_in, plan.C))
    _expect(w, "w", "float32", (E, plan.n_paths, plan.C))
    _expect(grad_out, "grad_out", "float32", (N, plan.dim_out, plan.C))
    dev = x.device
    if "x" in want and grad_x is None:
        grad_x = torch.empty((N, plan.dim_in, plan.C), device=dev, dtype=torch.float32)
    if "w" in want and grad_w is None:
        grad_w = torch.empty((E, plan.n_paths, plan.C), device=dev, dtype=torch.float32)
    if "r" in want and grad_r is None:
        grad_r = torch.empty((E, 3), device=dev, dtype=torch.float32)
    _expect(grad_x, "grad_x", "float32", (N, plan.dim_in, plan.C))
    _expect(grad_w, "grad_w", "float32", (E, plan.n_paths, plan.C))
    _expect(grad_r, "grad_r", "float32", (E, 3))
    dev = _need_cuda(row_ptr, src, rev_ptr, rev_perm, dst, r, frames, x, w, grad_out, grad_x, grad_w, grad_r)
    workspace = _tp_workspace(plan, N, E, False, workspace, dev)
    _need_cuda(x, workspace)
    _launch(dev, "etp_backward", _load().etp_backward, plan.handle, N, E, _ptr(row_ptr), _ptr(src), _ptr(rev_ptr),
            _ptr(rev_perm), _ptr(dst), _ptr(r), _ptr(frames), _ptr(x), _ptr(w), _ptr(grad_out), _ptr(grad_x),
            _ptr(grad_w), _ptr(grad_r), _ptr(workspace), workspace.numel(), stream=stream)
    return grad_x, grad_w, grad_r


def cart_forward(plan: Plan, row_ptr, src, r, x, w, out=None, workspace=None, stream=None):
    """Cartesian edge convolution (launches etp_cart_forward): x and out in independent STF components."""
    import torch

    N, E = row_ptr.numel() - 1, src.numel()
    _check_graph(row_ptr, src, N, E)
    _expect(r, "r", "float32", (E, 3))
    _expect(x, "x", "float32", (N, plan.dim_in, plan.C))
    _expect(w, "w", "float32", (E, plan.n_paths, plan.C))
    if out is None:
        out = torch.empty((N, plan.dim_out, plan.C), device=x.device, dtype=torch.float32)
    _expect(out, "out", "float32", (N, plan.dim_out, plan.C))
    dev = _need_cuda(row_ptr, src, r, x, w, out)
    workspace = _tp_workspace(plan, N, E, False, workspace, dev)
    _need_cuda(out, workspace)
    _launch(dev, "etp_cart_forward", _load().etp_cart_forward, plan.handle, N, E, _ptr(row_ptr), _ptr(src), _ptr(r),
            _ptr(x), _ptr(w), _ptr(out), _ptr(workspace), workspace.numel(), stream=stream)
    return out


def node_product(plan: Plan, x, w, K=None, cartesian=False, out=None, stream=None):
    """Node-local product of correlation order K (launches etp_node_product): out = B(K) with
    B(1) = x, B(k+1) = sum_p w[k-1, p] couple_p(B(k), x). x [N, D, C]; w [K-1, P, C] (K defaults
    to w.shape[0] + 1; w may be None for K = 1); spherical or Cartesian (independent STF
    components) couplings."""
    import torch

    N = x.shape[0] if x.dim() == 3 else -1
    _expect(x, "x", "float32", (N, plan.dim_in, plan.C))
    if K is None:
        if w is None:
            raise ValueError("give K or w")
        K = w.shape[0] + 1
    if K < 1:
        raise ValueError(f"K must be >= 1, got {K}")
    if K > 1:
        if w is None:
            raise ValueError("w is required for K > 1")
        _expect(w, "w", "float32", (K - 1, plan.n_paths, plan.C))
    if out is None:
        out = torch.empty((N, plan.dim_out, plan.C), device=x.device, dtype=torch.float32)
    _expect(out, "out", "float32", (N, plan.dim_out, plan.C))
    for t in (x, w if K > 1 else None):
        if t is not None and t.numel() and out.numel() and \
                out.data_ptr() < t.data_ptr() + 4 * t.numel() and t.data_ptr() < out.data_ptr() + 4 * out.numel():
            raise ValueError("out must not overlap x or w")
    dev = _need_cuda(x, out, *([w] if K > 1 else []))
    _launch(dev, "etp_node_product", _load().etp_node_product, plan.handle, N, int(K), int(bool(cartesian)),
            _ptr(x), _ptr(w) if K > 1 else None, _ptr(out), stream=stream)
    return out


def node_product_ops(plan: Plan, cartesian=False) -> int:
    """FP32 operations per node, channel and step of the node-local product kernel."""
    n = ctypes.c_int()
    _check(_load().etp_node_product_ops(plan.handle, int(bool(cartesian)), ctypes.byref(n)), "node product ops")
    return n.value


def cart_backward(plan: Plan, row_ptr, src, rev_ptr, rev_perm, dst, r, x, w, grad_out, want=("x", "w", "r"),
                  workspace=None, stream=None):
    """VJP of cart_forward (launches etp_cart_backward): (grad_x, grad_w, grad_r), unwanted ones None."""
    import torch

    N, E = row_ptr.numel() - 1, src.numel()
    _check_graph(row_ptr, src, N, E)
    _expect(rev_ptr, "rev_ptr", "int32", (N + 1,))
    _expect(rev_perm, "rev_perm", "int32", (E,))
    _expect(dst, "dst", "int32", (E,))
    _expect(r, "r", "float32", (E, 3))
    _expect(x, "x", "float32", (N, plan.dim_in, plan.C))
    _expect(w, "w", "float32", (E, plan.n_paths, plan.C))
    _expect(grad_out, "grad_out", "float32", (N, plan.dim_out, plan.C))
    dev = x.device
    gx = torch.empty((N, plan.dim_in, plan.C), device=dev, dtype=torch.float32) if "x" in want else None
    gw = torch.empty((E, plan.n_paths, plan.C), device=dev, dtype=torch.float32) if "w" in want else None
    gr = torch.empty((E, 3), device=dev, dtype=torch.float32) if "r" in want else None
    dev = _need_cuda(row_ptr, src, rev_ptr, rev_perm, dst, r, x, w, grad_out, gx, gw, gr)
    workspace = _tp_workspace(plan, N, E, False, workspace, dev)
    _need_cuda(x, workspace)
    _launch(dev, "etp_cart_backward", _load().etp_cart_backward, plan.handle, N, E, _ptr(row_ptr), _ptr(src),
            _ptr(rev_ptr), _ptr(rev_perm), _ptr(dst), _ptr(r), _ptr(x), _ptr(w), _ptr(grad_out), _ptr(gx), _ptr(gw),
            _ptr(gr), _ptr(workspace), workspace.numel(), stream=stream)
    return gx, gw, gr


def double_backward(plan: Plan, row_ptr, src, rev_ptr, rev_perm, dst, r, x, w, grad_out, gg_x=None, gg_w=None,
                    gg_r=None, want=("g", "x", "w", "r"), out=None, workspace=None, stream=None):
    """VJP of the VJP (launches etp_double_backward): dict with 'grad_g', 'grad_x', 'grad_w', 'grad_r'
    (the wanted ones) of <gg_x, grad_x> + <gg_w, grad_w> + <gg_r, grad_r>; None cotangents are zero."""
    import torch

    N, E = row_ptr.numel() - 1, src.numel()
    _check_graph(row_ptr, src, N, E)
    _expect(rev_ptr, "rev_ptr", "int32", (N + 1,))
    _expect(rev_perm, "rev_perm", "int32", (E,))
    _expect(dst, "dst", "int32", (E,))
    _expect(r, "r", "float32", (E, 3))
    for t, name in ((x, "x"), (gg_x, "gg_x")):
        _expect(t, name, "float32", (N, plan.dim_in, plan.C))
    for t, name in ((w, "w"), (gg_w, "gg_w")):
        _expect(t, name, "float32", (E, plan.n_paths, plan.C))
    _expect(grad_out, "grad_out", "float32", (N, plan.dim_out, plan.C))
    _expect(gg_r, "gg_r", "float32", (E, 3))
    shapes = {"g": (N, plan.dim_out, plan.C), "x": (N, plan.dim_in, plan.C), "w": (E, plan.n_paths, plan.C),
              "r": (E, 3)}
    out = dict(out or {})
    for k in "gxwr":
        key = "grad_" + k
        if k in want and out.get(key) is None:
            out[key] = torch.empty(shapes[k], device=x.device, dtype=torch.float32)
        _expect(out.get(key), key, "float32", shapes[k])
    dev = _need_cuda(row_ptr, src, rev_ptr, rev_perm, dst, r, x, w, grad_out, gg_x, gg_w, gg_r, *out.values())
    workspace = _tp_workspace(plan, N, E, False, workspace, dev)
    _need_cuda(x, workspace)
    _launch(dev, "etp_double_backward", _load().etp_double_backward, plan.handle, N, E, _ptr(row_ptr), _ptr(src),
            _ptr(rev_ptr), _ptr(rev_perm), _ptr(dst), _ptr(r), _ptr(x), _ptr(w), _ptr(grad_out), _ptr(gg_x),
            _ptr(gg_w), _ptr(gg_r), _ptr(out.get("grad_g")), _ptr(out.get("grad_x")), _ptr(out.get("grad_w")),
            _ptr(out.get("grad_r")), _ptr(workspace), workspace.numel(), stream=stream)
    return out


def assemble_forces(N: int, row_ptr, rev_ptr, rev_perm, grad_r, r=None, forces=None, virial=None, stream=None):
    """(forces [N, 3], virial [N, 3, 3] or None) from grad_r = dE/dr (etp_assemble_forces).
    The per-atom virial is computed when r is given."""
    import torch

    _expect(grad_r, "grad_r", "float32", (None, 3))
    E = grad_r.shape[0]
    _expect(row_ptr, "row_ptr", "int32", (N + 1,))
    _expect(rev_ptr, "rev_ptr", "int32", (N + 1,))
    _expect(rev_perm, "rev_perm", "int32", (E,))
    _expect(r, "r", "float32", (E, 3))
    dev = grad_r.device
    if forces is None:
        forces = torch.empty((N, 3), device=dev, dtype=torch.float32)
    if r is not None and virial is None:
        virial = torch.empty((N, 3, 3), device=dev, dtype=torch.float32)
    _expect(forces, "forces", "float32", (N, 3))
    if virial is not None and (str(virial.dtype) != "torch.float32" or virial.numel() != 9 * N):
        raise ValueError("virial: expected float32 with N*9 elements")
    dev = _need_cuda(row_ptr, rev_ptr, rev_perm, grad_r, r, forces, virial)
    _launch(dev, "etp_assemble_forces", _load().etp_assemble_forces, int(N), int(E), _ptr(row_ptr), _ptr(rev_ptr),
            _ptr(rev_perm), _ptr(r), _ptr(grad_r), _ptr(forces), _ptr(virial), stream=stream)
    return forces, virial


def radial_workspace_size(plan: Plan, E: int, n_basis: int, hidden: int) -> int:
    b = ctypes.c_size_t()
    _check(_load().etp_radial_workspace_size(plan.handle, int(E), int(n_basis), int(hidden), ctypes.byref(b)),
           "etp_radial_workspace_size")
    return b.value


def _radial_ws(plan, E, W1, workspace):
    import torch

    nbytes = radial_workspace_size(plan, E, W1.shape[0], W1.shape[1])
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=W1.device)
    _expect(workspace, "workspace", "uint8", (None,))
    return workspace


def radial_forward(plan: Plan, r, W1, W2, r_cut: float, w=None, workspace=None, stream=None):
    """w [E, P, C] = SiLU(bessel(|r|) W1) W2 (etp_radial_forward)."""
    import torch

    _expect(r, "r", "float32", (None, 3))
    E = r.shape[0]
    _expect(W1, "W1", "float32", (None, None))
    _expect(W2, "W2", "float32", (W1.shape[1], plan.n_paths * plan.C))
    if w is None:
        w = torch.empty((E, plan.n_paths, plan.C), device=r.device, dtype=torch.float32)
    _expect(w, "w", "float32", (E, plan.n_paths, plan.C))
    workspace = _radial_ws(plan, E, W1, workspace)
    dev = _need_cuda(r, W1, W2, w, workspace)
    _launch(dev, "etp_radial_forward", _load().etp_radial_forward, plan.handle, E, W1.shape[0], W1.shape[1],
            float(r_cut), _ptr(r), _ptr(W1), _ptr(W2), _ptr(w), _ptr(workspace), workspace.numel(), stream=stream)
    return w


def radial_backward(plan: Plan, r, W1, W2, r_cut: float, grad_w, grad_r, grad_W1=None, grad_W2=None,
                    workspace=None, stream=None):
    """(grad_W1, grad_W2); adds the derivative through |r| to grad_r in place (etp_radial_backward)."""
    import torch

    _expect(r, "r", "float32", (None, 3))
    E = r.shape[0]
    _expect(W1, "W1", "float32", (None, None))
    _expect(W2, "W2", "float32", (W1.shape[1], plan.n_paths * plan.C))
    _expect(grad_w, "grad_w", "float32", (E, plan.n_paths, plan.C))
    _expect(grad_r, "grad_r", "float32", (E, 3))
    if grad_W1 is None:
        grad_W1 = torch.empty_like(W1)
    if grad_W2 is None:
        grad_W2 = torch.empty_like(W2)
    _expect(grad_W1, "grad_W1", "float32", tuple(W1.shape))
    _expect(grad_W2, "grad_W2", "float32", tuple(W2.shape))
    workspace = _radial_ws(plan, E, W1, workspace)
    dev = _need_cuda(r, W1, W2, grad_w, grad_r, grad_W1, grad_W2, workspace)
    _launch(dev, "etp_radial_backward", _load().etp_radial_backward, plan.handle, E, W1.shape[0], W1.shape[1],
            float(r_cut), _ptr(r), _ptr(W1), _ptr(W2), _ptr(grad_w), _ptr(grad_W1), _ptr(grad_W2), _ptr(grad_r),
            _ptr(workspace), workspace.numel(), stream=stream)
    return grad_W1, grad_W2


def fused_workspace_size(plan: Plan, E: int, n_basis: int = 8, hidden: int = 64) -> int:
    b = ctypes.c_size_t()
    _check(_load().etp_fused_workspace_size(plan.handle, int(E), int(n_basis), int(hidden), ctypes.byref(b)),
           "etp_fused_workspace_size")
    return b.value


def fused_forward(plan: Plan, row_ptr, src, r, x, W1, W2, r_cut: float, out=None, workspace=None, stream=None):
    """out [N, D, C] = forward(plan, ..., w = radial_forward(plan, r, W1, W2, r_cut)) without storing w
    (launches etp_fused_forward)."""
    import torch

    N, E = row_ptr.numel() - 1, src.numel()
    _check_graph(row_ptr, src, N, E)
    _expect(r, "r", "float32", (E, 3))
    _expect(x, "x", "float32", (N, plan.dim_in, plan.C))
    _expect(W1, "W1", "float32", (None, None))
    _expect(W2, "W2", "float32", (W1.shape[1], plan.n_paths * plan.C))
    if out is None:
        out = torch.empty((N, plan.dim_out, plan.C), device=x.device, dtype=torch.float32)
    _expect(out, "out", "float32", (N, plan.dim_out, plan.C))
    nbytes = fused_workspace_size(plan, E, W1.shape[0], W1.shape[1])
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _expect(workspace, "workspace", "uint8", (None,))
    dev = _need_cuda(row_ptr, src, r, x, W1, W2, out, workspace)
    _launch(dev, "etp_fused_forward", _load().etp_fused_forward, plan.handle, N, E, _ptr(row_ptr), _ptr(src),
            _ptr(r), _ptr(x), W1.shape[0], W1.shape[1], float(r_cut), _ptr(W1), _ptr(W2), _ptr(out),
            _ptr(workspace), workspace.numel(), stream=stream)
    return out


def reverse_csr_workspace_size(N: int, E: int) -> int:
    b = ctypes.c_size_t()
    _check(_load().etp_reverse_csr_workspace_size(int(N), int(E), ctypes.byref(b)), "workspace_size")
    return b.value


def build_reverse_csr(N: int, row_ptr, src, with_dst=True, workspace=None, stream=None):
    """(rev_ptr [N+1], rev_perm [E], dst [E] or None), all int32 on the device (etp_build_reverse_csr)."""
    import torch

    E = src.numel()
    _check_graph(row_ptr, src, N, E)
    dev = row_ptr.device
    rev_ptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
    rev_perm = torch.empty(E, dtype=torch.int32, device=dev)
    dst = torch.empty(E, dtype=torch.int32, device=dev) if with_dst else None
    nbytes = reverse_csr_workspace_size(N, E)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    _expect(workspace, "workspace", "uint8", (None,))
    dev = _need_cuda(row_ptr, src, rev_ptr, rev_perm, dst, workspace)
    _launch(dev, "etp_build_reverse_csr", _load().etp_build_reverse_csr, N, E, _ptr(row_ptr), _ptr(src),
            _ptr(rev_ptr), _ptr(rev_perm), _ptr(dst), _ptr(workspace), workspace.numel(), stream=stream)
    return rev_ptr, rev_perm, dst


def build_reverse_csr_static(N: int, row_ptr, src, with_dst=True, stream=None):
    """As build_reverse_csr, with the library's fixed device scratch instead of a workspace
    (etp_build_reverse_csr_static; N, E <= 2^18; calls that overlap on the GPU race)."""
    import torch

    E = src.numel()
    _check_graph(row_ptr, src, N, E)
    dev = row_ptr.device
    rev_ptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
    rev_perm = torch.empty(E, dtype=torch.int32, device=dev)
    dst = torch.empty(E, dtype=torch.int32, device=dev) if with_dst else None
    dev = _need_cuda(row_ptr, src, rev_ptr, rev_perm, dst)
    _launch(dev, "etp_build_reverse_csr_static", _load().etp_build_reverse_csr_static, N, E, _ptr(row_ptr),
            _ptr(src), _ptr(rev_ptr), _ptr(rev_perm), _ptr(dst), stream=stream)
    return rev_ptr, rev_perm, dst


class Schedule:
    """Locality schedule of a CSR graph (etp_build_locality_schedule): node order, the
    forward CSR over that order (ord_ptr, ord_edge), the reverse CSR over that order
    (rev_ptr, rev_perm) and the destination of every edge, all int32 on the device."""

    def __init__(self, N, E, order, ord_ptr, ord_edge, rev_ptr, rev_perm, dst):
        self.N, self.E = N, E
        self.order, self.ord_ptr, self.ord_edge = order, ord_ptr, ord_edge
        self.rev_ptr, self.rev_perm, self.dst = rev_ptr, rev_perm, dst

    def tensors(self):
        return self.order, self.ord_ptr, self.ord_edge, self.rev_ptr, self.rev_perm, self.dst


def locality_schedule_workspace_size(N: int, E: int) -> int:
    b = ctypes.c_size_t()
    _check(_load().etp_locality_schedule_workspace_size(int(N), int(E), ctypes.byref(b)), "workspace_size")
    return b.value


def locality_schedule(N: int, row_ptr, src, pos, cell: float, out: Schedule = None, workspace=None, stream=None):
    """Schedule whose rows follow the Morton order of the nodes' cells (side `cell`) of pos [N, 3]
    (etp_build_locality_schedule). out: a Schedule of the same sizes to overwrite."""
    import torch

    E = src.numel()
    _check_graph(row_ptr, src, N, E)
    _expect(pos, "pos", "float32", (N, 3))
    dev = row_ptr.device
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = Schedule(N, E, torch.empty(N, **i32), torch.empty(N + 1, **i32), torch.empty(E, **i32),
                       torch.empty(N + 1, **i32), torch.empty(E, **i32), torch.empty(E, **i32))
    if (out.N, out.E) != (N, E):
        raise ValueError(f"schedule for (N, E) = {(out.N, out.E)}, graph has {(N, E)}")
    nbytes = locality_schedule_workspace_size(N, E)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    _expect(workspace, "workspace", "uint8", (None,))
    dev = _need_cuda(row_ptr, src, pos, workspace, *out.tensors())
    _launch(dev, "etp_build_locality_schedule", _load().etp_build_locality_schedule, N, E, _ptr(row_ptr), _ptr(src),
            _ptr(pos), float(cell), *[_ptr(t) for t in out.tensors()], _ptr(workspace), workspace.numel(),
            stream=stream)
    return out


def forward_ordered(plan: Plan, sched: Schedule, src, r, x, w, out=None, frames=None, workspace=None, stream=None):
    """forward() on a locality schedule (etp_forward_ordered): the same out, rows visited in schedule order."""
    import torch

    N, E = sched.N, sched.E
    _expect(src, "src", "int32", (E,))
    _expect(r, "r", "float32", (E, 3))
    _expect(frames, "frames", "float32", (E, FRAME_FLOATS))
    _expect(x, "x", "float32", (N, plan.dim_in, plan.C))
    _expect(w, "w", "float32", (E, plan.n_paths, plan.C))
    if out is None:
        out = torch.empty((N, plan.dim_out, plan.C), device=x.device, dtype=torch.float32)
    _expect(out, "out", "float32", (N, plan.dim_out, plan.C))
    dev = _need_cuda(sched.order, sched.ord_ptr, sched.ord_edge, src, r, frames, x, w, out)
    workspace = _tp_workspace(plan, N, E, True, workspace, dev)
    _need_cuda(out, workspace)
    _launch(dev, "etp_forward_ordered", _load().etp_forward_ordered, plan.handle, N, E, _ptr(sched.order),
            _ptr(sched.ord_ptr), _ptr(sched.ord_edge), _ptr(src), _ptr(r), _ptr(frames), _ptr(x), _ptr(w),
            _ptr(out), _ptr(workspace), workspace.numel(), stream=stream)
    return out


def backward_ordered(plan: Plan, sched: Schedule, r, x, w, grad_out, want=("x", "w", "r"), grad_x=None,
                     grad_w=None, grad_r=None, frames=None, workspace=None, stream=None):
    """backward() on a locality schedule (etp_backward_ordered): the same (grad_x, grad_w, grad_r)."""
    import torch

    N, E = sched.N, sched.E
    _expect(r, "r", "float32", (E, 3))
    _expect(frames, "frames", "float32", (E, FRAME_FLOATS))
    _expect(x, "x", "float32", (N, plan.dim_in, plan.C))
    _expect(w, "w", "float32", (E, plan.n_paths, plan.C))
    _expect(grad_out, "grad_out", "float32", (N, plan.dim_out, plan.C))
    dev = x.device
    if "x" in want and grad_x is None:
        grad_x = torch.empty((N, plan.dim_in, plan.C), device=dev, dtype=torch.float32)
    if "w" in want and grad_w is None:
        grad_w = torch.empty((E, plan.n_paths, plan.C), device=dev, dtype=torch.float32)
    if "r" in want and grad_r is None:
        grad_r = torch.empty((E, 3), device=dev, dtype=torch.float32)
    _expect(grad_x, "grad_x", "float32", (N, plan.dim_in, plan.C))
    _expect(grad_w, "grad_w", "float32", (E, plan.n_paths, plan.C))
    _expect(grad_r, "grad_r", "float32", (E, 3))
    dev = _need_cuda(sched.order, sched.rev_ptr, sched.rev_perm, sched.dst, r, frames, x, w, grad_out, grad_x,
                     grad_w, grad_r)
    workspace = _tp_workspace(plan, N, E, True, workspace, dev)
    _need_cuda(x, workspace)
    _launch(dev, "etp_backward_ordered", _load().etp_backward_ordered, plan.handle, N, E, _ptr(sched.order),
            _ptr(sched.rev_ptr), _ptr(sched.rev_perm), _ptr(sched.dst), _ptr(r), _ptr(frames), _ptr(x), _ptr(w),
            _ptr(grad_out), _ptr(grad_x), _ptr(grad_w), _ptr(grad_r), _ptr(workspace), workspace.numel(),
            stream=stream)
    return grad_x, grad_w, grad_r


def device_fault() -> int:
    """1 if a bounded wait inside a kernel ran out since the last call (never expected); clears it."""
    f = ctypes.c_int()
    _check(_load().etp_device_fault(ctypes.byref(f)), "etp_device_fault")
    return f.value


def validate_csr(N: int, row_ptr, src, stream=None) -> int:
    """The ETP_CSR_* bits of every problem found in the CSR (0 = valid). Synchronises the stream."""
    import torch

    _check_graph(row_ptr, src, N, src.numel())
    flag = torch.empty(1, dtype=torch.int32, device=row_ptr.device)
    dev = _need_cuda(row_ptr, src, flag)
    _launch(dev, "etp_validate_csr", _load().etp_validate_csr, N, src.numel(), _ptr(row_ptr), _ptr(src),
            _ptr(flag), stream=stream)
    return int(flag.item())
