"""Python front-end of libmuon over torch tensors.

PyTorch provides device memory and streams only; ``MuonPlan`` passes raw
pointers, shapes and the current CUDA stream to the C ABI.

    plan = MuonPlan([W.shape for W in weights], zero_momentum_of=[M...])
    plan.step(list(zip(weights, grads, moms)), lr=4.2e-4, weight_decay=0.1)

The hybrid split of "Muon is Scalable for LLM Training" (Sec. 2.2) sends the
parameters that are not matrices (RMSNorm gains, embedding, LM head) to
AdamW with the same learning rate and weight decay; ``AdamWPlan`` does that
step for them.

    adam = AdamWPlan([g.numel() for g in gains], states=[(m, v) ...])
    adam.step(list(zip(gains, grads, ms, vs)), step=t, lr=4.2e-4, weight_decay=0.1)

``HybridStep`` runs both plans as one optimizer step.

Sec. 3.4 compares optimisers by the SVD entropy of the weight matrices;
``EntropyPlan`` computes it on the GPU.

    ent = EntropyPlan([W.shape for W in weights])
    H = ent.compute(weights)            # fp32 [n] on the device
"""

from __future__ import annotations

import ctypes

import torch

from . import _lib as L

DEFAULT_COEFFS = (3.4445, -4.7750, 2.0315)


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _check_tensor(t: torch.Tensor, dtype, name: str, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


_GDT = {torch.bfloat16: L.MUON_DT_BF16, torch.float32: L.MUON_DT_FP32}


class MuonPlan:
    """A libmuon plan for a fixed list of matrix shapes on the current device."""

    def __init__(self, shapes, *, momenta=None, fp32_ns: bool = False, max_workspace_bytes: int | None = None,
                 stream=None):
        shapes = [tuple(int(v) for v in s) for s in shapes]
        if any(len(s) != 2 for s in shapes):
            raise ValueError("Muon plans take 2-D shapes only")
        self.shapes = shapes
        self.n = len(shapes)
        arr = (L.muon_param_t * self.n)()
        flags = L.MUON_INIT_FP32_NS if fp32_ns else 0
        if momenta is not None:
            flags |= L.MUON_INIT_ZERO_MOMENTUM
            for i, M in enumerate(momenta):
                _check_tensor(M, torch.float32, f"M[{i}]", shapes[i])
                arr[i].M = M.data_ptr()
        for i, (r, c) in enumerate(shapes):
            arr[i].rows, arr[i].cols = r, c
        if max_workspace_bytes:
            self._plan = L.muon_init_ex(arr, self.n, flags | L.MUON_INIT_MAX_WORKSPACE, int(max_workspace_bytes),
                                        _stream_handle(stream))
        else:
            self._plan = L.muon_init(arr, self.n, flags, _stream_handle(stream))
        self._params = (L.muon_param_t * self.n)()
        self._key = None
        self._bound = {}   # recent bindings: key -> descriptor array
        self._x = (ctypes.c_void_p * self.n)()
        self._o = (ctypes.c_void_p * self.n)()

    # ------------------------------------------------------------ the step
    def bind(self, params):
        """Fill the descriptor array from [(W, G, M), ...].  The last few
        distinct bindings are kept, so alternating between buffer sets (double
        buffered gradients) costs no re-validation.  A binding is reused only
        when every tensor has the same address, shape, dtype and contiguity
        (which fix its layout), so another tensor or a view at a cached
        address is validated afresh."""
        if len(params) != self.n:
            raise ValueError(f"expected {self.n} (W, G, M) triples, got {len(params)}")
        key = tuple((W.data_ptr(), G.data_ptr(), M.data_ptr(), W.shape, G.shape, M.shape, W.dtype, G.dtype, M.dtype,
                     W.is_contiguous(), G.is_contiguous(), M.is_contiguous()) for W, G, M in params)
        if key == self._key:
            return
        cached = self._bound.get(key)
        if cached is not None:
            self._params, self._key = cached, key
            return
        arr = (L.muon_param_t * self.n)()
        for i, (W, G, M) in enumerate(params):
            shp = self.shapes[i]
            _check_tensor(W, torch.float32, f"W[{i}]", shp)
            _check_tensor(G, (torch.bfloat16, torch.float32), f"G[{i}]", shp)
            _check_tensor(M, torch.float32, f"M[{i}]", shp)
            d = arr[i]
            d.W, d.G, d.M = W.data_ptr(), G.data_ptr(), M.data_ptr()
            d.rows, d.cols = shp
            d.g_dtype = _GDT[G.dtype]
            d.reserved = 0
        if len(self._bound) >= 4:
            self._bound.pop(next(iter(self._bound)))
        self._bound[key] = arr
        self._params, self._key = arr, key

    def step(self, params=None, *, lr: float, weight_decay: float, momentum: float = 0.95, ns_steps: int = 5,
             coeffs=DEFAULT_COEFFS, rms_scale: float = 0.2, nesterov: bool = True, precision: str = "bf16",
             update_rms: torch.Tensor | None = None, scale: str = "max_dim", hidden_dim: float = 0.0,
             stream=None) -> None:
        """One Muon step over every matrix (in place on W and M).

        `scale` picks how O is scaled (Sec. 3.1): "max_dim" rms_scale sqrt(max(A, B))
        (Eq. 4), "hidden" rms_scale sqrt(hidden_dim) (Eq. 5) or "update_norm"
        rms_scale / RMS(O) (Eq. 6)."""
        modes = {"max_dim": L.MUON_SCALE_MAX_DIM, "hidden": L.MUON_SCALE_HIDDEN,
                 "update_norm": L.MUON_SCALE_UPDATE_NORM}
        if scale not in modes:
            raise ValueError(f"scale must be one of {sorted(modes)}")
        if params is not None:
            self.bind(params)
        elif self._key is None:
            raise ValueError("no parameters bound")
        hp = L.muon_hparams_t(lr, weight_decay, momentum, int(ns_steps), coeffs[0], coeffs[1], coeffs[2],
                              rms_scale, 1 if nesterov else 0,
                              L.MUON_NS_FP32 if precision == "fp32" else L.MUON_NS_BF16, modes[scale],
                              float(hidden_dim))
        rms_ptr = None
        if update_rms is not None:
            _check_tensor(update_rms, torch.float32, "update_rms", (self.n,))
            rms_ptr = update_rms.data_ptr()
        L.muon_step(self._plan, self._params, self.n, hp, rms_ptr, _stream_handle(stream))

    def orthogonalize(self, xs, outs, *, ns_steps: int = 5, coeffs=DEFAULT_COEFFS, precision: str = "bf16",
                      stream=None) -> None:
        """outs[i] = Newton-Schulz(xs[i]) (fp32 outputs) for every matrix."""
        if len(xs) != self.n or len(outs) != self.n:
            raise ValueError("one input and one output per planned matrix")
        dt = None
        for i, (x, o) in enumerate(zip(xs, outs)):
            _check_tensor(x, (torch.bfloat16, torch.float32), f"X[{i}]", self.shapes[i])
            _check_tensor(o, torch.float32, f"O[{i}]", self.shapes[i])
            if dt is None:
                dt = x.dtype
            elif x.dtype != dt:
                raise TypeError("all inputs of one call share a dtype")
            self._x[i] = x.data_ptr()
            self._o[i] = o.data_ptr()
        L.muon_orthogonalize(self._plan, self._x, self._o, self.n, _GDT[dt], ns_steps, coeffs,
                             L.MUON_NS_FP32 if precision == "fp32" else L.MUON_NS_BF16, _stream_handle(stream))

    # ------------------------------------------------------------ bookkeeping
    @property
    def workspace_bytes(self) -> int:
        return L.muon_workspace_bytes(self._plan)

    @property
    def waves(self) -> int:
        """How many waves a call runs (1 unless the plan has a workspace cap)."""
        return L.muon_num_waves(self._plan)

    def status(self) -> int:
        """Synchronizing read-and-clear of the device status (an int status code)."""
        return L.muon_get_status(self._plan)

    def profile(self, enable: bool = True, spans: bool = False) -> None:
        """Record phase times of the following calls: an event after every
        launch, or with spans=True only where the kernel class changes (the
        Newton-Schulz chain of each wave as one span, phase newton_schulz)."""
        mode = 0 if not enable else (L.MUON_PROFILE_SPANS if spans else L.MUON_PROFILE_LAUNCHES)
        L.muon_profile_enable(self._plan, mode)

    def profile_read(self):
        ms, cnt, calls = L.muon_profile_read(self._plan)
        return {"ms": dict(zip(L.PHASE_NAMES, ms)), "launches": dict(zip(L.PHASE_NAMES, cnt)), "calls": calls}

    def close(self) -> None:
        if getattr(self, "_plan", None):
            L.muon_destroy(self._plan)
            self._plan = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class AdamWPlan:
    """A libmuon AdamW plan for a fixed list of tensors (sizes and gradient
    dtypes) on the current device."""

    def __init__(self, numels, *, g_dtypes=None, states=None, stream=None):
        self.numels = [int(v) for v in numels]
        self.n = len(self.numels)
        self.g_dtypes = list(g_dtypes) if g_dtypes is not None else [torch.bfloat16] * self.n
        arr = (L.muon_adamw_param_t * self.n)()
        flags = 0
        if states is not None:
            flags |= L.MUON_INIT_ZERO_MOMENTUM
            for i, (m, v) in enumerate(states):
                _check_tensor(m, torch.float32, f"m[{i}]")
                _check_tensor(v, torch.float32, f"v[{i}]")
                arr[i].m, arr[i].v = m.data_ptr(), v.data_ptr()
        for i, e in enumerate(self.numels):
            arr[i].numel = e
            arr[i].g_dtype = _GDT[self.g_dtypes[i]]
            arr[i].decay = 1
        self._plan = L.muon_adamw_init(arr, self.n, flags, _stream_handle(stream))
        self._params = (L.muon_adamw_param_t * self.n)()

    def step(self, tensors, *, step: int, lr: float, weight_decay: float, betas=(0.9, 0.95), eps: float = 1e-8,
             decay=None, stream=None) -> None:
        """One AdamW step: tensors = [(P, G, m, v), ...] in plan order; `decay`
        (list of bools, default all True) selects the tensors that get weight
        decay."""
        if len(tensors) != self.n:
            raise ValueError("one (P, G, m, v) per planned tensor")
        for i, (P, G, m, v) in enumerate(tensors):
            e = self.numels[i]
            _check_tensor(P, torch.float32, f"P[{i}]")
            _check_tensor(G, self.g_dtypes[i], f"G[{i}]")
            _check_tensor(m, torch.float32, f"m[{i}]")
            _check_tensor(v, torch.float32, f"v[{i}]")
            if not (P.numel() == G.numel() == m.numel() == v.numel() == e):
                raise ValueError(f"tensor {i} does not have {e} elements")
            a = self._params[i]
            a.P, a.G, a.m, a.v = P.data_ptr(), G.data_ptr(), m.data_ptr(), v.data_ptr()
            a.numel = e
            a.g_dtype = _GDT[self.g_dtypes[i]]
            a.decay = 1 if (decay is None or decay[i]) else 0
        hp = L.muon_adamw_hparams_t(lr, betas[0], betas[1], eps, weight_decay, int(step))
        L.muon_adamw_step(self._plan, self._params, self.n, hp, _stream_handle(stream))

    def close(self) -> None:
        if getattr(self, "_plan", None):
            L.muon_adamw_destroy(self._plan)
            self._plan = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class PackPlan:
    """One-launch copy of a fixed list of (src, dst) tensor pairs (bf16 or
    fp32 each; the values are converted when the dtypes differ)."""

    def __init__(self, pairs, *, stream=None):
        pairs = list(pairs)
        if not pairs:
            raise ValueError("a pack plan needs at least one (src, dst) pair")
        arr = (L.muon_segment_t * len(pairs))()
        for k, (src, dst) in enumerate(pairs):
            for t, name in ((src, "src"), (dst, "dst")):
                _check_tensor(t, (torch.bfloat16, torch.float32), f"{name}[{k}]")
            if src.numel() != dst.numel():
                raise ValueError(f"pair {k}: {src.numel()} source and {dst.numel()} destination elements")
            a = arr[k]
            a.src, a.dst, a.numel = src.data_ptr(), dst.data_ptr(), src.numel()
            a.src_dtype, a.dst_dtype = _GDT[src.dtype], _GDT[dst.dtype]
        self._keep = pairs  # the plan holds raw pointers: keep the tensors alive
        self._plan = L.muon_pack_init(arr, len(pairs), _stream_handle(stream))

    def run(self, stream=None) -> None:
        L.muon_pack_run(self._plan, _stream_handle(stream))

    def close(self) -> None:
        if getattr(self, "_plan", None):
            L.muon_pack_destroy(self._plan)
            self._plan = None
            self._keep = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class HybridStep:
    """The full optimizer step of "Muon is Scalable for LLM Training"
    (Sec. 2.2, "Matching update RMS of AdamW"): Muon for every matrix
    parameter and AdamW for the rest (RMSNorm gains, embedding, LM head), one
    learning rate and one weight decay for both; the RMSNorm gains keep their
    weight decay (Appendix D, "Training stability").  Both plans enqueue on
    the same stream, Muon first; nothing waits on the host.

        opt = HybridStep([W.shape for W in mats], [p.numel() for p in vecs],
                         momenta=Ms, adam_states=[(m, v), ...])
        opt.step(list(zip(mats, mat_grads, Ms)), list(zip(vecs, vec_grads, ms, vs)),
                 t=step, lr=4.2e-4, weight_decay=0.1)
    """

    def __init__(self, matrix_shapes, vector_numels, *, momenta=None, adam_states=None, vector_g_dtypes=None,
                 vector_decay=None, max_workspace_bytes: int | None = None, stream=None):
        self.muon = MuonPlan(matrix_shapes, momenta=momenta, max_workspace_bytes=max_workspace_bytes, stream=stream)
        self.adamw = AdamWPlan(vector_numels, g_dtypes=vector_g_dtypes, states=adam_states, stream=stream)
        self.vector_decay = list(vector_decay) if vector_decay is not None else None

    def step(self, matrices, vectors, *, t: int, lr: float, weight_decay: float, momentum: float = 0.95,
             ns_steps: int = 5, coeffs=DEFAULT_COEFFS, betas=(0.9, 0.95), eps: float = 1e-8,
             update_rms: torch.Tensor | None = None, stream=None) -> None:
        """matrices: [(W, G, M), ...] in the Muon plan's order; vectors:
        [(P, G, m, v), ...] in the AdamW plan's order; t >= 1 is the step
        count of AdamW's bias corrections."""
        self.muon.step(matrices, lr=lr, weight_decay=weight_decay, momentum=momentum, ns_steps=ns_steps,
                       coeffs=coeffs, update_rms=update_rms, stream=stream)
        self.adamw.step(vectors, step=t, lr=lr, weight_decay=weight_decay, betas=betas, eps=eps,
                        decay=self.vector_decay, stream=stream)

    def status(self) -> int:
        return self.muon.status()

    def close(self) -> None:
        self.muon.close()
        self.adamw.close()


class EntropyPlan:
    """A libmuon SVD-entropy plan for a fixed list of fp32 matrix shapes on the
    current device (Sec. 3.4): H = -(1/log n) sum p_i log p_i with
    p_i = sigma_i^2 / sum sigma_j^2 over the n = min(rows, cols) singular values."""

    _PHASES = ("gram", "tridiagonal", "bisection", "entropy")

    def __init__(self, shapes, *, stream=None):
        self.shapes = [tuple(int(v) for v in s) for s in shapes]
        if any(len(s) != 2 for s in self.shapes):
            raise ValueError("entropy plans take 2-D shapes only")
        self.n = len(self.shapes)
        self._plan = L.muon_entropy_init(self.shapes, _stream_handle(stream))
        self.num_singular_values = L.muon_entropy_num_singular_values(self._plan)
        # CTAs per matrix in the tridiagonal reduction (a cluster per matrix)
        self.cluster_size = L.muon_entropy_cluster_size(self._plan)
        self._w = (ctypes.c_void_p * self.n)()

    def compute(self, weights, H=None, sigma=None, *, stream=None) -> torch.Tensor:
        """Entropy of each matrix into H (fp32 [n] on the device, allocated if
        None).  sigma, if given (fp32 [num_singular_values]), receives each
        matrix's singular values, descending, matrix after matrix."""
        if len(weights) != self.n:
            raise ValueError(f"expected {self.n} matrices, got {len(weights)}")
        for i, W in enumerate(weights):
            _check_tensor(W, torch.float32, f"W[{i}]", self.shapes[i])
            self._w[i] = W.data_ptr()
        if H is None:
            H = torch.empty(self.n, dtype=torch.float32, device=weights[0].device)
        _check_tensor(H, torch.float32, "H", (self.n,))
        sp = None
        if sigma is not None:
            _check_tensor(sigma, torch.float32, "sigma", (self.num_singular_values,))
            sp = sigma.data_ptr()
        L.muon_entropy_compute(self._plan, self._w, self.n, H.data_ptr(), sp, _stream_handle(stream))
        return H

    def status(self):
        """(status code, per matrix of the last call 1 if its eigenvalues were
        computed and 0 if it was non-finite); synchronising."""
        return L.muon_entropy_get_status(self._plan, self.n)

    def profile(self, enable: bool = True) -> None:
        L.muon_entropy_profile(self._plan, enable)

    def profile_read(self) -> dict:
        return dict(zip(self._PHASES, L.muon_entropy_profile(self._plan, True, read=True)))

    def close(self) -> None:
        if getattr(self, "_plan", None):
            L.muon_entropy_destroy(self._plan)
            self._plan = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
