"""Host-side checks of the vector-parameter step's C ABI (dion_vec_*): defaults and
argument validation return the documented codes before any device work (no GPU)."""
import ctypes

import pytest

import rank_orthonormalized_optimizer_b200 as dion

FAKE = 1 << 20          # an aligned address that is never dereferenced


def _opts(which="adamw", **kw):
    o = dion.vec_default_options(which)
    for k, v in kw.items():
        setattr(o, k, v)
    return o


def _tensors(*specs):
    arr = (dion.VecTensor * max(len(specs), 1))()
    for i, (x, g, m, v, n) in enumerate(specs):
        arr[i].x, arr[i].g, arr[i].m, arr[i].v, arr[i].numel = x, g, m, v, n
    return arr


def _call(arr, n, o):
    return dion.dion_vec_step(arr, n, ctypes.byref(o) if o is not None else None, None)


def test_defaults():
    a = dion.vec_default_options("adamw")
    assert (a.rule, a.step) == (0, 1)
    assert abs(a.lr - 1e-3) < 1e-10 and abs(a.beta1 - 0.9) < 1e-7 and abs(a.beta2 - 0.999) < 1e-7
    assert abs(a.eps - 1e-8) < 1e-15 and abs(a.weight_decay - 0.01) < 1e-9
    l = dion.vec_default_options("lion")
    assert l.rule == 1 and abs(l.lr - 1e-4) < 1e-11 and abs(l.beta2 - 0.99) < 1e-7
    assert l.weight_decay == 0.0
    o = dion.VecOptions()
    assert dion.dion_vec_default_options(7, ctypes.byref(o)) == dion.ERR_INVALID_ARG
    assert dion.dion_vec_default_options(0, None) == dion.ERR_INVALID_ARG


@pytest.mark.parametrize("field,value", [("rule", 2), ("lr", float("nan")), ("beta1", 1.0),
                                         ("beta2", -0.5), ("eps", 0.0), ("step", 0),
                                         ("weight_decay", -1.0),
                                         ("weight_decay", float("inf"))])
def test_adamw_option_checks(field, value):
    arr = _tensors((FAKE, FAKE, FAKE, FAKE, 16))
    assert _call(arr, 1, _opts(**{field: value})) == dion.ERR_INVALID_ARG
    assert dion.dion_last_error()


def test_lion_ignores_eps_step_and_v():
    # eps and step are AdamW's; v may be NULL for Lion: valid arguments reach the device
    arr = _tensors((FAKE, FAKE, FAKE, None, 16))
    code = _call(arr, 1, _opts("lion", eps=0.0, step=0))
    assert code in (dion.ERR_CUDA, dion.ERR_DEVICE, dion.OK)
    assert code != dion.ERR_INVALID_ARG


def test_tensor_checks():
    o = _opts()
    assert _call(None, 0, None) == dion.ERR_INVALID_ARG
    assert _call(None, 2, o) == dion.ERR_INVALID_ARG
    assert _call(_tensors((FAKE, FAKE, FAKE, FAKE, 4)), -1, o) == dion.ERR_INVALID_ARG
    assert _call(_tensors((FAKE, FAKE, FAKE, FAKE, -4)), 1, o) == dion.ERR_INVALID_ARG
    assert _call(_tensors((FAKE, None, FAKE, FAKE, 4)), 1, o) == dion.ERR_INVALID_ARG
    assert _call(_tensors((FAKE, FAKE, FAKE, None, 4)), 1, o) == dion.ERR_INVALID_ARG
    assert _call(_tensors((FAKE + 2, FAKE, FAKE, FAKE, 4)), 1, o) == dion.ERR_MISALIGNED
    assert _call(_tensors((FAKE, FAKE, FAKE, FAKE + 1, 4)), 1, o) == dion.ERR_MISALIGNED
    # the second tensor is checked too, before anything runs
    two = _tensors((FAKE, FAKE, FAKE, FAKE, 4), (FAKE, FAKE, None, FAKE, 4))
    assert _call(two, 2, o) == dion.ERR_INVALID_ARG


def test_empty_tensors_need_no_pointers():
    # numel 0 with NULL pointers is accepted (a 4-byte-aligned, non-16-byte-aligned
    # tensor beside it is valid too); the call then reaches the device check
    arr = _tensors((None, None, None, None, 0), (FAKE + 4, FAKE + 4, FAKE + 4, FAKE + 4, 5))
    try:
        import torch
        no_gpu = not torch.cuda.is_available()
    except Exception:
        no_gpu = True
    if no_gpu:
        assert _call(arr, 2, _opts()) in (dion.ERR_CUDA, dion.ERR_DEVICE)
        assert dion.dion_vec_last_launch_count() == 0


def test_plan_checks_its_tensors_on_the_host():
    """VecStepPlan refuses what the C ABI could not take, before any call: CPU tensors,
    other dtypes, non-contiguous views, mismatched sizes and list lengths."""
    import torch
    x = torch.zeros(8)
    with pytest.raises(ValueError, match="CUDA"):
        dion.VecStepPlan([x], [x.clone()], [x.clone()], [x.clone()])
    with pytest.raises(ValueError, match="one entry per parameter"):
        dion.VecStepPlan([x, x], [x], [x], [x])
    with pytest.raises(KeyError):
        dion.VecStepPlan([x], [x], [x], [x], rule="sgd")
