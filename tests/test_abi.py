"""The C-ABI library: loads, exports every function include/*.h declares, and
validates configurations on the host (no GPU needed for any of this)."""
import ctypes
import os
import re

import pytest

from synth_inputs import make_config, workload, WORKLOADS


def _declared(repo_root):
    names = set()
    for f in os.listdir(os.path.join(repo_root, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(repo_root, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            for m in re.finditer(r"\b(ttt_[a-z0-9_]+)\s*\(", text):
                names.add(m.group(1))
    return names


def test_library_exports_every_declared_function(repo_root):
    from weight_sequence_mixing_b200 import binding
    names = _declared(repo_root)
    assert {"ttt_create", "ttt_forward", "ttt_destroy", "ttt_workspace_size"} <= names
    lib = ctypes.CDLL(binding._LIB_PATH)
    for n in sorted(names):
        assert hasattr(lib, n), n
    assert names <= set(binding.EXPORTED)


def _create(cfg_c):
    from weight_sequence_mixing_b200 import binding
    h = ctypes.c_void_p()
    st = binding.LIB.ttt_create(ctypes.byref(cfg_c), ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_every_workload_configuration_is_accepted(name):
    from weight_sequence_mixing_b200 import binding
    cfg = workload(name)
    st, h = _create(binding.make_config(cfg))
    assert st == 0, binding.status_string(st)
    P = binding.LIB.ttt_param_count(h)
    expect = ({"linear": 1, "mlp2_gelu": 2, "swiglu": 3, "glu": 2}[cfg["inner"]] * cfg["d"] * cfg["h"]
              if cfg["inner"] != "dwconv" else cfg["d"] * cfg["ksize"] ** 2)
    assert P == expect
    assert binding.LIB.ttt_workspace_size(h) >= 256
    assert binding.LIB.ttt_host_staging_size(h) > 0
    binding.LIB.ttt_destroy(h)


@pytest.mark.parametrize("bad", [
    dict(B=0), dict(H=0), dict(N=0), dict(Nq=0), dict(d=0), dict(causal=1, Nq=7),
])
def test_invalid_configurations_are_rejected(bad):
    from weight_sequence_mixing_b200 import binding
    kw = dict(N=16, d=64, h=128, dtype="bf16")
    kw.update(bad)
    c = binding.make_config(make_config(**kw))
    st, h = _create(c)
    assert st == binding.TTT_ERR_INVALID_ARG and not h.value


def test_invalid_enum_and_flag_values_are_rejected():
    from weight_sequence_mixing_b200 import binding
    for field, value in (("inner", 7), ("loss", -1), ("loss", 3), ("opt", 9), ("dtype", 5), ("flags", 128), ("ns_iters", -1),
                         ("epochs", -1), ("epochs", 65)):
        c = binding.make_config(make_config(N=16, d=64, h=128))
        setattr(c, field, value)
        st, h = _create(c)
        assert st == binding.TTT_ERR_INVALID_ARG, field


@pytest.mark.parametrize("inner", ["linear", "mlp2_gelu", "swiglu"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_first_layer_only_is_accepted_and_leaves_the_plan_alone(inner, dtype):
    from weight_sequence_mixing_b200 import binding
    kw = dict(N=300, d=128, h=128, inner=inner, loss="neg_dot", dtype=dtype, opt="momentum_muon",
              weight_l2norm=True)
    sizes = []
    for flo in (False, True):
        c = binding.make_config(make_config(first_layer_only=flo, **kw))
        assert bool(c.flags & binding.FLAG_FIRST_LAYER_ONLY) == flo
        st, h = _create(c)
        assert st == 0, binding.status_string(st)
        sizes.append((binding.LIB.ttt_param_count(h), binding.LIB.ttt_workspace_size(h)))
        binding.LIB.ttt_destroy(h)
    assert sizes[0] == sizes[1]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("opt", ["gd", "momentum", "muon", "momentum_muon"])
def test_momentum_state_size(dtype, opt):
    from weight_sequence_mixing_b200 import binding
    B, H, d, h = 2, 3, 128, 256
    cfg = make_config(B=B, H=H, N=300, d=d, h=h, inner="swiglu", loss="neg_dot", dtype=dtype, opt=opt)
    st, hd = _create(binding.make_config(cfg))
    assert st == 0
    n = binding.LIB.ttt_state_size(hd)
    binding.LIB.ttt_destroy(hd)
    if opt in ("gd", "muon"):
        assert n == 0
    else:  # the momentum of every matrix of every (batch entry, head), fp32
        assert n == B * H * 3 * d * h * 4
    # the blob does not depend on the token counts, chunking or flags
    st, hd = _create(binding.make_config(dict(cfg, N=1000, Nq=40, chunk=256, weight_l2norm=True,
                                              w0_per_batch=True)))
    assert st == 0 and binding.LIB.ttt_state_size(hd) == n
    binding.LIB.ttt_destroy(hd)


def test_forward_state_checks_state_alignment_without_touching_the_gpu():
    from weight_sequence_mixing_b200 import binding
    st, h = _create(binding.make_config(make_config(N=16, d=64, h=128, opt="momentum")))
    assert st == 0
    lib = binding.LIB
    fake = ctypes.c_void_p(4096)
    bad = ctypes.c_void_p(4096 + 4)
    for a, b in ((bad, None), (None, bad)):
        assert lib.ttt_forward_state(h, fake, fake, fake, None, fake, fake, None, a, b, fake, 1 << 30,
                                     None) == binding.TTT_ERR_INVALID_ARG
    assert lib.ttt_forward_state(h, None, fake, fake, None, fake, fake, None, None, None, fake, 1 << 30,
                                 None) == binding.TTT_ERR_INVALID_ARG
    lib.ttt_destroy(h)


@pytest.mark.parametrize("inner", ["linear", "mlp2_gelu", "swiglu"])
def test_rmse_loss_is_built_where_mse_is(inner):
    from weight_sequence_mixing_b200 import binding
    for dtype in ("f32", "bf16"):
        for loss in ("mse", "rmse"):
            st, h = _create(binding.make_config(make_config(N=300, d=128, h=128, inner=inner, loss=loss,
                                                            dtype=dtype)))
            if dtype == "bf16" and inner == "swiglu":
                assert st == binding.TTT_ERR_UNSUPPORTED and not h.value
            else:
                assert st == 0, binding.status_string(st)
                binding.LIB.ttt_destroy(h)


def _dw(**kw):
    base = dict(B=2, H=3, N=20, d=64, inner="dwconv", loss="neg_dot", opt="gd", dtype="bf16", grid_h=4, grid_w=5)
    base.update(kw)
    return make_config(**base)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("k", [1, 3, 5, 7])
def test_dwconv_configuration_is_accepted(dtype, k):
    from weight_sequence_mixing_b200 import binding
    st, h = _create(binding.make_config(_dw(dtype=dtype, ksize=k, opt="momentum", loss="mse", weight_l2norm=True)))
    assert st == 0, binding.status_string(st)
    assert binding.LIB.ttt_param_count(h) == 64 * k * k
    assert binding.LIB.ttt_state_size(h) == 2 * 3 * 64 * k * k * 4
    binding.LIB.ttt_destroy(h)
    assert binding.plan_info(_dw(dtype=dtype, ksize=k))["path"] == 2


@pytest.mark.parametrize("bad,status", [
    (dict(grid_w=4), "invalid"), (dict(ksize=2), "invalid"), (dict(ksize=9), "invalid"), (dict(grid_h=0), "invalid"),
    (dict(Nq=10), "invalid"), (dict(causal=1), "unsupported"), (dict(chunk=10), "unsupported"),
    (dict(key_instnorm=True), "unsupported"), (dict(loss="rmse"), "unsupported"), (dict(opt="muon"), "unsupported"),
    (dict(opt="momentum_muon"), "unsupported"),
])
def test_dwconv_configurations_outside_the_built_set_are_rejected(bad, status):
    from weight_sequence_mixing_b200 import binding
    st, h = _create(binding.make_config(_dw(**bad)))
    want = binding.TTT_ERR_INVALID_ARG if status == "invalid" else binding.TTT_ERR_UNSUPPORTED
    assert st == want and not h.value


@pytest.mark.parametrize("d,ok", [(64, False), (192, False), (128, True), (256, True)])
def test_bf16_linear_model_needs_whole_128_row_gradient_tiles(d, ok):
    # d = 64 once divided by zero in the gradient-shape heuristic (a crash of ttt_create)
    from weight_sequence_mixing_b200 import binding
    st, h = _create(binding.make_config(make_config(N=500, d=d, inner="linear", dtype="bf16", loss="neg_dot")))
    assert st == (0 if ok else binding.TTT_ERR_UNSUPPORTED)
    if ok:
        binding.LIB.ttt_destroy(h)
    st, h = _create(binding.make_config(make_config(N=500, d=d, inner="linear", dtype="f32", loss="neg_dot")))
    assert st == 0
    binding.LIB.ttt_destroy(h)


def test_forward_rejects_null_and_small_workspace_without_touching_the_gpu():
    from weight_sequence_mixing_b200 import binding
    st, h = _create(binding.make_config(make_config(N=16, d=64, h=128)))
    assert st == 0
    lib = binding.LIB
    fake = ctypes.c_void_p(4096)
    assert lib.ttt_forward(h, None, fake, fake, None, fake, fake, None, fake, 1 << 30, None) == binding.TTT_ERR_INVALID_ARG
    assert lib.ttt_forward(h, fake, fake, fake, None, fake, fake, None, fake, 16, None) == binding.TTT_ERR_WORKSPACE
    misaligned = ctypes.c_void_p(4096 + 8)
    assert lib.ttt_forward(h, misaligned, fake, fake, None, fake, fake, None, fake, 1 << 30, None) == binding.TTT_ERR_INVALID_ARG
    lib.ttt_destroy(h)


def test_status_strings():
    from weight_sequence_mixing_b200 import binding
    for s in range(-6, 1):
        assert binding.status_string(s) and binding.status_string(s) != "unknown status"
    assert binding.status_string(-99) == "unknown status"


def test_binding_config_struct_matches_the_c_header(tmp_path, repo_root):
    # the ctypes mirror of ttt_config must have the C layout: compare sizeof and every
    # field offset with a C program compiled against include/ttt.h
    import ctypes
    import shutil
    import subprocess

    from weight_sequence_mixing_b200 import binding

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    names = [f[0] for f in binding.TTTConfig._fields_]
    src = tmp_path / "layout.c"
    # (ttt_diag.h includes ttt.h: both headers must be plain C)
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"ttt_diag.h\"\nint main(void) {\n"
                   + "  printf(\"%zu\\n\", sizeof(ttt_config));\n"
                   + "".join(f"  printf(\"%zu\\n\", offsetof(ttt_config, {n}));\n" for n in names)
                   + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.join(repo_root, "include"), str(src), "-o", str(exe)], check=True)
    out = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert out[0] == ctypes.sizeof(binding.TTTConfig)
    assert out[1:] == [getattr(binding.TTTConfig, n).offset for n in names]


def test_binding_refuses_buffers_of_the_wrong_size_dtype_or_place():
    # the library reads and writes buffers by the configured sizes: the binding checks them first
    import torch

    from weight_sequence_mixing_b200 import binding
    cfg = make_config(B=2, H=3, N=40, Nq=24, d=64, h=128, inner="swiglu", loss="neg_dot", dtype="bf16",
                      eta_mode="per_token")
    layer = binding.TTTLayer(cfg, device="cpu")
    P = layer.P
    ok = dict(Q=torch.zeros(2, 3, 24, 64, dtype=torch.bfloat16), K=torch.zeros(2, 3, 40, 64, dtype=torch.bfloat16),
              V=torch.zeros(2, 3, 40, 64, dtype=torch.bfloat16), eta=torch.zeros(2, 3, 40),
              W0=torch.zeros(3, P), O=torch.zeros(2, 3, 24, 64, dtype=torch.bfloat16), W_out=torch.zeros(2, 3, P))
    layer.check_buffers("cpu", **ok)  # right sizes on the host: accepted
    layer.check_buffers("cpu", **dict(ok, eta=None, W_out=None))
    bad = [dict(K=torch.zeros(2, 3, 39, 64, dtype=torch.bfloat16)), dict(Q=torch.zeros(2, 3, 24, 64)),
           dict(eta=torch.zeros(2, 3, 40, dtype=torch.float64)), dict(W0=torch.zeros(2, 3, P)),
           dict(O=torch.zeros(2, 3, 64, 24, dtype=torch.bfloat16).transpose(2, 3)), dict(V=None)]
    for b in bad:
        with pytest.raises(ValueError):
            layer.check_buffers("cpu", **dict(ok, **b))
    with pytest.raises(ValueError):
        layer.check_buffers("cuda", **ok)  # host tensors where device memory is expected
    layer.close()
    # one state per batch entry: W0 is [B, H, P]
    per = binding.TTTLayer(dict(cfg, w0_per_batch=True), device="cpu")
    per.check_buffers("cpu", **dict(ok, W0=torch.zeros(2, 3, P)))
    with pytest.raises(ValueError):
        per.check_buffers("cpu", **ok)
    per.close()


def test_every_entry_point_refuses_a_null_handle_or_buffer_without_gpu_work():
    import ctypes

    from weight_sequence_mixing_b200 import binding
    lib = binding.LIB
    inv = binding.TTT_ERR_INVALID_ARG
    fake = ctypes.c_void_p(4096)
    assert lib.ttt_create(None, None) == inv
    out = ctypes.c_void_p(1234)
    assert lib.ttt_create(None, ctypes.byref(out)) == inv and not out.value  # *out cleared
    assert lib.ttt_param_count(None) == 0 and lib.ttt_workspace_size(None) == 0
    assert lib.ttt_state_size(None) == 0 and lib.ttt_host_staging_size(None) == 0
    assert lib.ttt_launch_count(None) == 0
    assert lib.ttt_forward(None, fake, fake, fake, None, fake, fake, None, fake, 1 << 30, None) == inv
    assert lib.ttt_forward_state(None, fake, fake, fake, None, fake, fake, None, None, None, fake, 1 << 30,
                                 None) == inv
    assert lib.ttt_forward_host(None, fake, fake, fake, None, fake, fake, None, fake, 1 << 30, fake, 1 << 30,
                                None) == inv
    assert lib.ttt_forward_noalloc(None, fake, fake, fake, None, fake, fake, None, None, None) == inv
    assert lib.ttt_query_status(None, fake, None) == inv
    assert lib.ttt_profile_enable(None, 1) == inv
    ms, cnt = (ctypes.c_float * 8)(), (ctypes.c_int * 8)()
    assert lib.ttt_profile_collect(None, 8, ms, cnt) == inv
    info = (ctypes.c_int * 7)()
    assert lib.ttt_plan_info(None, info, 7) == inv
    assert lib.ttt_selftest_timeout(None, None) == inv
    assert lib.ttt_selftest_activation(3, 16, fake, fake, fake, None) == inv  # unknown kind
    assert lib.ttt_selftest_activation(-1, 16, fake, fake, fake, None) == inv
    assert lib.ttt_selftest_activation(0, 16, None, fake, fake, None) == inv
    assert lib.ttt_selftest_activation(0, -1, fake, fake, fake, None) == inv
    assert lib.ttt_selftest_activation(0, 0, None, None, None, None) == 0  # nothing to do
    assert lib.ttt_selftest_gemm(2, 0, 0, 64, 128, 64, 64, 1, 1, None, fake, fake, None) == inv
    lib.ttt_destroy(None)  # a no-op
    assert lib.ttt_stage_name(99) == b"unknown"
    # a real handle: null outputs and a null workspace are refused too
    st, h = _create(binding.make_config(make_config(N=16, d=64, h=128)))
    assert st == 0
    assert lib.ttt_query_status(h, None, None) == inv
    assert lib.ttt_profile_collect(h, 0, ms, cnt) == inv and lib.ttt_plan_info(h, None, 7) == inv
    assert lib.ttt_forward_host(h, fake, fake, fake, None, fake, None, None, fake, 1 << 30, fake, 1 << 30,
                                None) == inv
    lib.ttt_destroy(h)
