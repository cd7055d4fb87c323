"""torch.optim-style front end over the C ABI.

``TwoStateOptimizer`` keeps, for every parameter, the fp32 state of the
32-bit two-state update (state1 = m, or [m1 | m2] for AdEMAMix; state2 = v)
and steps each parameter group with ONE launch of the library's kernel,
whatever the number, sizes and dtypes (fp32/fp16/bf16) of its tensors.  The
classes mirror the optimizer families of the bitsandbytes issue "Investigate
a 256-thread SM103 path for small 32-bit optimizer tensors" (section "B300
benchmark and acceptance": AdamW32bit and AdEMAMix32bit).

flatten=True moves the parameters of each (param group, device, dtype) into
one flat buffer (each parameter's .data becomes a view of it), points every
.grad at a view of a matching flat gradient buffer, and keeps the state flat
as well; step() is then one call per flat buffer with no per-parameter
Python work, and zero_grad() zeroes the flat gradients in place (gradients
must keep accumulating into those views: do not replace p.grad).  Results are
the same bits as without flattening, since the update is elementwise.

max_unorm > 0 bounds each parameter's update norm by max_unorm times its
weight norm (opt2s_step_max_unorm: four launches per group and step).  With
flatten=True the bound still applies per parameter: the flat buffers are
stepped through one record per parameter, and AdEMAMix keeps each
parameter's [m1 | m2] together in the flat state.  It is not combined with
capturable=True.

lamb=True makes the step LAMB's (opt2s_step_lamb; You et al. 2020,
Algorithm 2; Adam moments only): per parameter, the Adam direction plus
weight_decay * param, scaled by the trust ratio ||param|| / ||direction||.
Like max_unorm it takes four launches per group and step, keeps one record
per parameter under flatten=True, and is not combined with capturable=True.

Without flatten, each group's launch records (the tensors' addresses) are
built once and refreshed in place every step by a small C++ helper
(csrc/opt2s_marshal.cpp) that reads the current parameter and gradient
addresses; a group is rebuilt only when a gradient is missing or a tensor no
longer fits its record.  zero_grad() zeroes gradients in place by default
(set_to_none=False), so that their addresses, and the library's cached plan,
stay the same.  Without the helper the records are reused while the tensors
are the same objects (checked by identity); reassigning a tensor's storage in
place (``p.data = x``) is then not seen: call refresh() after it.  A group
shares one step count (one launch, one set of bias corrections): a parameter
left out of a step, its gradient None, still counts that step.

AdamW8bit, Adam8bit and AdEMAMix8bit keep 8-bit blockwise state
(opt2s_step_8bit) for parameters of at least ``min_8bit_size`` elements and
fp32 state for the smaller ones, one launch per group
(TwoStateOptimizer8bit).

load_state_dict keeps each state tensor's own dtype (fp32 moments of 16-bit
parameters, uint8 codes), where torch.optim's loader alone would cast them to
the parameter's dtype; with flatten=True it copies the loaded state into the
flat buffers the steps read.  The per-parameter state keys differ between
the layouts (state1/state2 without flatten; exp_avg, exp_avg_sq and
exp_avg_slow, views of the flat buffers, with it), so a state dict loads into
an optimizer of the same layout.

capturable=True routes every step through opt2s_plan_step_table: the per-step
scalars live in a device table and the step index in device memory, so
``step()`` may be captured in a CUDA graph and each replay performs the next
step.  Make one eager ``step()`` before capturing (it builds the launch plan),
and call ``refill_step_table()`` between replays at least once every
``table_len`` steps (``steps_left()`` tells how many remain); the table holds
the hyper-parameters of the refill, so a change of ``lr`` or another group
setting takes effect at the next refill.
"""
from __future__ import annotations

import contextlib
import ctypes
import importlib.machinery
import importlib.util
import operator
import os

import torch

from . import binding as B

_marshal = None


def _marshal_module():
    """The in-tree marshalling extension (csrc/opt2s_marshal.cpp, built by
    _build.build), or None when it has not been built: the identity check in
    Python then stands in for it (same results, more host time)."""
    global _marshal
    if _marshal is None:
        from . import _build
        path = _build.marshal_path()
        _marshal = False
        if os.path.exists(path):
            loader = importlib.machinery.ExtensionFileLoader(_build.MARSHAL_NAME, path)
            spec = importlib.util.spec_from_loader(_build.MARSHAL_NAME, loader)
            mod = importlib.util.module_from_spec(spec)
            loader.exec_module(mod)
            _marshal = mod
    return _marshal or None


def _on_device(index):
    """Makes CUDA device `index` current for a launch (nothing to do when it
    already is): the library plans and launches on the current device."""
    if index == torch._C._cuda_getDevice():
        return contextlib.nullcontext()
    return torch.cuda.device(index)


class TwoStateOptimizer(torch.optim.Optimizer):
    def __init__(self, params, algo: str = "adamw", lr: float = 1e-3,
                 betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
                 beta3: float = 0.9999, alpha: float = 5.0, skip_zeros: bool = False,
                 capturable: bool = False, table_len: int = 1024, flatten: bool = False,
                 max_unorm: float = 0.0, lamb: bool = False):
        if algo not in B.ALGOS:
            raise ValueError(f"algo must be one of {sorted(B.ALGOS)}")
        if not (0.0 <= max_unorm < float("inf")):
            raise ValueError("max_unorm must be finite and >= 0 (0 disables the bound)")
        if max_unorm > 0.0 and capturable:
            raise ValueError("max_unorm and capturable are not combined")
        if lamb and (capturable or max_unorm > 0.0 or algo == "ademamix"):
            raise ValueError("lamb takes Adam moments and is not combined with capturable "
                             "or max_unorm")
        defaults = dict(lr=lr, betas=tuple(betas), eps=eps, weight_decay=weight_decay,
                        beta3=beta3, alpha=alpha, skip_zeros=skip_zeros)
        self.algo = "ademamix" if algo == "ademamix" else "adam"
        self.capturable = capturable
        self.table_len = int(table_len)
        self.max_unorm = float(max_unorm)
        self.lamb = bool(lamb)
        super().__init__(params, defaults)
        self._group_cache = {}
        self._flat = None
        if flatten:
            if capturable:
                raise ValueError("flatten and capturable are not combined")
            self._flatten()

    # ---- flat layout ---------------------------------------------------------
    def _flatten(self):
        self._flat = []
        two = self.algo == "ademamix"
        for gi, group in enumerate(self.param_groups):
            by_kind = {}
            for p in group["params"]:
                if not p.is_cuda:
                    raise ValueError("parameters must be CUDA tensors")
                by_kind.setdefault((p.device, p.dtype), []).append(p)
            for (dev, dt), ps in by_kind.items():
                n = sum(p.numel() for p in ps)
                fp = torch.empty(n, dtype=dt, device=dev)
                fg = torch.zeros(n, dtype=dt, device=dev)
                fs1 = torch.zeros(2 * n if two else n, dtype=torch.float32, device=dev)
                fs2 = torch.zeros(n, dtype=torch.float32, device=dev)
                # per_param: one record per parameter (needed by the per-
                # parameter norms of max_unorm and LAMB); AdEMAMix then keeps
                # each parameter's [m1 | m2] together, else all m1 before all m2
                per_param = self.max_unorm > 0.0 or self.lamb
                off = 0
                views = ([], [], [], [])
                counter = torch.tensor(0, dtype=torch.int64)     # the entry's shared step count
                with torch.no_grad():
                    for p in ps:
                        k = p.numel()
                        fp[off:off + k].copy_(p.detach().reshape(-1))
                        if p.grad is not None:
                            fg[off:off + k].copy_(p.grad.detach().reshape(-1))
                        p.data = fp[off:off + k].view_as(p)
                        p.grad = fg[off:off + k].view_as(p)
                        st = self.state[p]
                        m1_at = 2 * off if (two and per_param) else off
                        st["exp_avg"] = fs1[m1_at:m1_at + k].view_as(p)
                        st["exp_avg_sq"] = fs2[off:off + k].view_as(p)
                        if two:
                            m2_at = m1_at + k if per_param else n + off
                            st["exp_avg_slow"] = fs1[m2_at:m2_at + k].view_as(p)
                        st["step"] = counter
                        views[0].append(fp[off:off + k])
                        views[1].append(fg[off:off + k])
                        views[2].append(fs1[m1_at:m1_at + (2 * k if two else k)])
                        views[3].append(fs2[off:off + k])
                        off += k
                entry = dict(group=gi, params=ps, param=fp, grad=fg, state1=fs1, state2=fs2, step=0,
                             counter=counter, device=dev.index,
                             views=[{key: self.state[p][key] for key in self.state[p] if key != "step"}
                                    for p in ps])
                if per_param:
                    entry["records"] = B.TensorList.from_tensors(*views)
                else:
                    tl = B.TensorList.from_tensors([fp], [fg], [fs1], [fs2])
                    with _on_device(dev.index):
                        entry["plan"] = B.Plan(tl, self.algo)
                self._flat.append(entry)

    @staticmethod
    def _check_flat_grads(f):
        """The flat layout steps its gradient buffer, so every parameter's
        .grad must still be its view into it.  Replacing the gradients (for
        instance module.zero_grad(), which sets them to None by default, and
        a backward that then makes new ones) would leave the buffer stale:
        the first and last parameters of each buffer are checked (O(1) per
        step) and the step refuses if either was replaced."""
        fg = f["grad"]
        base = fg.data_ptr()
        end = base + fg.numel() * fg.element_size()
        for p in (f["params"][0], f["params"][-1]):
            g = p.grad
            if g is None or not base <= g.data_ptr() < end:     # no other tensor lies in the buffer
                raise RuntimeError(
                    "flatten=True: a parameter's .grad is no longer its view of the flat gradient "
                    "buffer (was it set to None, e.g. by module.zero_grad()?); use the optimizer's "
                    "zero_grad(), which zeroes the views in place")

    def add_param_group(self, param_group):
        if getattr(self, "_flat", None) is not None:
            raise ValueError("flatten=True lays out the groups given at construction; add groups "
                             "before flattening, or use flatten=False")
        super().add_param_group(param_group)

    def zero_grad(self, set_to_none: bool = False):
        """Zero the gradients in place (one launch per device and dtype), so
        that the cached launch records stay valid; set_to_none=True drops
        them as torch.optim does (the next step then rebuilds the records)."""
        if self._flat is None:
            if set_to_none:
                return super().zero_grad(True)
            grads = [p.grad for g in self.param_groups for p in g["params"] if p.grad is not None]
            if grads:
                torch._foreach_zero_(grads)
            return None
        for f in self._flat:           # keep the views: gradients accumulate into them
            f["grad"].zero_()

    def refresh(self) -> None:
        """Forget the cached launch records (after ``p.data = x`` or another
        in-place change of a tensor's storage)."""
        for data in self._group_cache.values():
            for st in data["states"]:
                st["step"] = data["step"]
        self._group_cache = {}

    def load_state_dict(self, state_dict) -> None:
        """torch.optim's loader casts every floating-point state tensor to its
        parameter's dtype; the state here keeps its own (fp32 moments, uint8
        codes), so after it each tensor is copied again from the saved one,
        dtype and bits kept, onto the parameter's device."""
        super().load_state_dict(state_dict)
        from itertools import chain
        saved_ids = chain.from_iterable(g["params"] for g in state_dict["param_groups"])
        current = chain.from_iterable(g["params"] for g in self.param_groups)
        for sid, p in zip(saved_ids, current):
            saved = state_dict["state"].get(sid)
            if not saved:
                continue
            st = self.state[p]
            for k, v in saved.items():
                if k != "step" and isinstance(v, torch.Tensor):
                    st[k] = v.to(device=p.device, copy=True)
        if self._flat is not None:
            # the steps use the flat buffers: copy the loaded state into their
            # views and put the views (and the entry's step count) back
            with torch.no_grad():
                for f in self._flat:
                    for p, views in zip(f["params"], f["views"]):
                        st = self.state[p]
                        for key, view in views.items():
                            if key in st:
                                view.copy_(st[key].reshape(view.shape))
                            st[key] = view
                        if "step" in st:
                            f["step"] = int(st["step"])
                        st["step"] = f["counter"]
                    f["counter"].fill_(f["step"])
        self._group_cache = {}

    # ---- per-group launch data ------------------------------------------
    def _hyper(self, group):
        b1, b2 = group["betas"]
        return B.make_hyper(self.algo, lr=group["lr"], beta1=b1, beta2=b2, eps=group["eps"],
                            weight_decay=group["weight_decay"], beta3=group["beta3"],
                            alpha=group["alpha"], skip_zeros=group["skip_zeros"])

    def _state_of(self, p):
        st = self.state[p]
        if "state1" not in st:
            n = p.numel()
            st["state1"] = torch.zeros(2 * n if self.algo == "ademamix" else n,
                                       dtype=torch.float32, device=p.device)
            st["state2"] = torch.zeros(n, dtype=torch.float32, device=p.device)
            st["step"] = 0
        return st

    def _launch_data(self, gi, group):
        params = group["params"]
        cached = self._group_cache.get(gi)
        if cached is not None and cached["dense"] and len(params) == len(cached["params"]):
            marshal = _marshal_module()
            if marshal is not None:
                # every parameter has a record: refresh the addresses in place
                rc = getattr(marshal, self._refresh_fn)(params, cached["records"], len(params))
                if rc == 0 or (rc == 1 and not self.capturable):
                    return cached
            elif (all(map(operator.is_, [p.grad for p in params], cached["all_grads"]))
                  and all(map(operator.is_, params, cached["params"]))):
                return cached      # the same tensors as last step: reuse the records
        data = self._build_launch_data(gi, group, cached)
        data["all_grads"] = [p.grad for p in params]
        data["dense"] = len(data["params"]) == len(params) and all(
            map(operator.is_, data["params"], params))
        data["records"] = ctypes.addressof(data["tl"]._arr)
        return data

    def _build_launch_data(self, gi, group, cached):
        ps = [p for p in group["params"] if p.grad is not None]
        for p in ps:
            if not p.is_cuda or not p.is_contiguous() or not p.grad.is_contiguous():
                raise ValueError("parameters and gradients must be contiguous CUDA tensors")
        if len({p.device for p in ps} | {p.grad.device for p in ps}) > 1:
            raise ValueError("a parameter group's tensors and gradients must be on one CUDA device")
        key = tuple((p.data_ptr(), p.grad.data_ptr(), p.numel()) for p in ps)
        if cached is not None and cached["key"] == key:
            return cached
        states = [self._state_of(p) for p in ps]
        tl = self._records(ps, states)
        data = {"key": key, "params": ps, "tl": tl, "states": states, "step": 0,
                "device": ps[0].device.index if ps else None}
        if cached is not None:
            data["step"] = cached["step"]
            data["counter"] = cached["counter"]
            current = {id(st) for st in states}
            for st in cached["states"]:      # a parameter that leaves the group keeps its count
                if id(st) not in current:
                    st["step"] = cached["step"]
        else:
            data["step"] = int(states[0]["step"]) if states else 0
            data["counter"] = torch.tensor(data["step"], dtype=torch.int64)
        # every stepped parameter's state["step"] is the group's shared counter
        for st in states:
            st["step"] = data["counter"]
        if self.capturable:
            with _on_device(data["device"] if ps else torch._C._cuda_getDevice()):
                data["plan"] = B.Plan(tl, self.algo)
            dev = ps[0].device if ps else torch.device("cuda")
            data["table"] = torch.empty(self.table_len * ctypes.sizeof(B.opt2s_step_scalars),
                                        dtype=torch.uint8, device=dev)
            data["index"] = torch.zeros(1, dtype=torch.int32, device=dev)
            self._refill(data, group)
        self._group_cache[gi] = data
        return data

    _refresh_fn = "refresh_records"     # the marshalling helper's refresh for these records

    def _records(self, ps, states):
        """The launch records of parameters ps with their states."""
        return B.TensorList.from_tensors(ps, [p.grad for p in ps], [s["state1"] for s in states],
                                         [s["state2"] for s in states])

    def _refill(self, data, group):
        first = data["step"] + 1
        raw = B.fill_step_scalars(self._hyper(group), first, self.table_len)
        host = torch.frombuffer(bytearray(raw), dtype=torch.uint8)
        data["table"].copy_(host)
        data["index"].zero_()
        data["table_first"] = first

    # ---- public API --------------------------------------------------------
    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        if self._flat is not None:
            for f in self._flat:
                self._check_flat_grads(f)
                hyper = self._hyper(self.param_groups[f["group"]])
                with _on_device(f["device"]):
                    if "records" in f and self.lamb:
                        B.opt2s_step_lamb(f["records"], hyper, f["step"] + 1)
                    elif "records" in f:
                        B.opt2s_step_max_unorm(f["records"], hyper, self.max_unorm, f["step"] + 1)
                    else:
                        f["plan"].step(hyper, f["step"] + 1)
                f["step"] += 1
                f["counter"].fill_(f["step"])
            return loss
        for gi, group in enumerate(self.param_groups):
            data = self._launch_data(gi, group)
            if not data["params"]:
                continue
            with _on_device(data["device"]):
                if self.capturable:
                    data["plan"].step_table(group["skip_zeros"], data["table"].data_ptr(),
                                            self.table_len, data["index"].data_ptr())
                else:
                    self._launch(data["tl"], self._hyper(group), data["step"] + 1)
            data["step"] += 1
            data["counter"].fill_(data["step"])   # the parameters' shared step count
        return loss

    def _launch(self, tl, hyper, step):
        """One step of a group's records (not capturable)."""
        if self.lamb:
            B.opt2s_step_lamb(tl, hyper, step)
        elif self.max_unorm > 0.0:
            B.opt2s_step_max_unorm(tl, hyper, self.max_unorm, step)
        else:
            B.opt2s_step(tl, hyper, step)

    def refill_step_table(self, next_step: int | None = None) -> None:
        """Capturable mode: rewrite the device tables so that the next step
        performed (eagerly or by a graph replay) is ``next_step`` (default:
        one past the steps recorded by eager calls).  Call it only while no
        replay is in flight."""
        for gi, group in enumerate(self.param_groups):
            data = self._group_cache.get(gi)
            if data is None or "table" not in data:
                continue
            if next_step is not None:
                data["step"] = next_step - 1
                data["counter"].fill_(data["step"])
            self._refill(data, group)

    def steps_left(self) -> int:
        """Capturable mode: table entries left before a refill is needed
        (reads the device index; synchronizes)."""
        left = []
        for data in self._group_cache.values():
            if "index" in data:
                i = int(data["index"].item())
                left.append(0 if i < 0 else self.table_len - i)
        return min(left) if left else 0


class AdamW32bit(TwoStateOptimizer):
    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=1e-2, **kw):
        super().__init__(params, "adamw", lr, betas, eps, weight_decay, **kw)


class Adam32bit(TwoStateOptimizer):
    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0, **kw):
        super().__init__(params, "adam", lr, betas, eps, weight_decay, **kw)


class AdEMAMix32bit(TwoStateOptimizer):
    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999, 0.9999), alpha=5.0, eps=1e-8,
                 weight_decay=1e-2, **kw):
        b1, b2, b3 = betas
        super().__init__(params, "ademamix", lr, (b1, b2), eps, weight_decay, beta3=b3,
                         alpha=alpha, **kw)


class LAMB32bit(TwoStateOptimizer):
    """LAMB (You et al. 2020, Algorithm 2) with fp32 state: the weight decay
    sits inside the trust-ratio scaled update."""

    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999), eps=1e-6, weight_decay=1e-2, **kw):
        super().__init__(params, "adam", lr, betas, eps, weight_decay, lamb=True, **kw)


class TwoStateOptimizer8bit(TwoStateOptimizer):
    """The two-state optimizer with 8-bit blockwise state (opt2s_step_8bit;
    Dettmers, Lewis, Shleifer & Zettlemoyer, "8-bit Optimizers via Block-wise
    Quantization", ICLR 2022).  A parameter of at least ``min_8bit_size``
    elements keeps its state as one byte per element and quantity (uint8
    codes: state1 = m, or [m1 | m2] for AdEMAMix; state2 = v) plus one fp32
    absmax per 2,048-element block and quantity (absmax1, absmax2); a smaller
    one keeps fp32 state as in the 32-bit classes.  Each parameter group is
    one launch, mixed 8-bit and fp32 state included.  The state starts at
    zero: the code of 0 (127 in the signed map of m and m2, 0 in the unsigned
    map of v) with absmax 0.  Records are refreshed each step as in the
    32-bit classes; flatten, capturable, max_unorm and LAMB are not offered
    with 8-bit state."""

    _refresh_fn = "refresh_records8"

    def __init__(self, params, algo: str = "adamw", lr: float = 1e-3, betas=(0.9, 0.999),
                 eps: float = 1e-8, weight_decay: float = 0.0, beta3: float = 0.9999,
                 alpha: float = 5.0, skip_zeros: bool = False, min_8bit_size: int = B.MIN_8BIT_SIZE):
        if int(min_8bit_size) < 1:
            raise ValueError("min_8bit_size must be >= 1")
        self.min_8bit_size = int(min_8bit_size)
        super().__init__(params, algo, lr, betas, eps, weight_decay, beta3=beta3, alpha=alpha,
                         skip_zeros=skip_zeros)

    def _state_of(self, p):
        st = self.state[p]
        if "state1" not in st:
            n = p.numel()
            two = self.algo == "ademamix"
            if B.state_bits_for(n, self.min_8bit_size) == 8:
                nb = (n + B.BLOCK8 - 1) // B.BLOCK8
                st["state1"] = torch.full((2 * n if two else n,), 127, dtype=torch.uint8, device=p.device)
                st["state2"] = torch.zeros(n, dtype=torch.uint8, device=p.device)
                st["absmax1"] = torch.zeros(2 * nb if two else nb, dtype=torch.float32, device=p.device)
                st["absmax2"] = torch.zeros(nb, dtype=torch.float32, device=p.device)
            else:
                st["state1"] = torch.zeros(2 * n if two else n, dtype=torch.float32, device=p.device)
                st["state2"] = torch.zeros(n, dtype=torch.float32, device=p.device)
            st["step"] = 0
        return st

    def _records(self, ps, states):
        return B.TensorList8.from_tensors(ps, [p.grad for p in ps], [s["state1"] for s in states],
                                          [s["state2"] for s in states],
                                          [s.get("absmax1") for s in states],
                                          [s.get("absmax2") for s in states])

    def _launch(self, tl, hyper, step):
        B.opt2s_step_8bit(tl, hyper, step)


class AdamW8bit(TwoStateOptimizer8bit):
    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=1e-2, **kw):
        super().__init__(params, "adamw", lr, betas, eps, weight_decay, **kw)


class Adam8bit(TwoStateOptimizer8bit):
    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0, **kw):
        super().__init__(params, "adam", lr, betas, eps, weight_decay, **kw)


class AdEMAMix8bit(TwoStateOptimizer8bit):
    def __init__(self, params, lr=1e-3, betas=(0.9, 0.999, 0.9999), alpha=5.0, eps=1e-8,
                 weight_decay=1e-2, **kw):
        b1, b2, b3 = betas
        super().__init__(params, "ademamix", lr, (b1, b2), eps, weight_decay, beta3=b3,
                         alpha=alpha, **kw)
