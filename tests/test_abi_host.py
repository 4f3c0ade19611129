"""C ABI checks that need no GPU: the library loads, exports every declared entry point, and
its host-only functions (partition, accounting, argument validation) behave."""
import ctypes
import os
import re
import subprocess

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def zero():
    import zero_sharded_optimizer_03_b200 as z  # built by conftest at session start
    return z


def declared_functions():
    text = open(os.path.join(ROOT, "include", "zero.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(zero3?_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["zero_partition", "zero_reduce_scatter", "zero_adam_shard", "zero_allgather",
                 "zero_step", "zero3_gather_layer", "zero_memory_estimate", "zero_comm_volume"]:
        assert must in names


def test_every_declared_symbol_is_exported(zero):
    out = subprocess.run(["nm", "-D", "--defined-only", zero.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(zero.LIB_PATH)
    for n in declared_functions():
        assert getattr(lib, n) is not None


def test_binding_constants_match_the_header(zero):
    """Every integer #define of include/zero.h has the same value in the Python binding."""
    text = open(os.path.join(ROOT, "include", "zero.h")).read()
    defines = dict(re.findall(r"#define\s+(ZERO_[A-Z0-9_]+)\s+\(?(-?\d+)\)?\s", text))
    assert len(defines) >= 15
    for name, value in defines.items():
        assert getattr(zero, name) == int(value), name
    assert zero.ZERO_NOALLOC_MAX_WINDOW == zero.ZERO_NOALLOC_MAX_CTAS * 2048


STRUCTS = ["zero_partition_t", "zero_hparams_t", "zero_step_result_t", "zero_state_t",
           "zero_mem_t", "zero_rs_summary_t", "zero_offload_state_t"]


def test_binding_structures_match_the_header_layout(zero, tmp_path):
    """The ctypes structures have the size and field offsets that a C compiler gives the
    header's structures (compiled here with gcc against include/zero.h)."""
    fields = {n: [f[0] for f in getattr(zero, n)._fields_] for n in STRUCTS}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "zero.h"', "int main(void) {"]
    for n in STRUCTS:
        lines.append('printf("%s size %%zu\\n", sizeof(%s));' % (n, n))
        for f in fields[n]:
            lines.append('printf("%s %s %%zu\\n", offsetof(%s, %s));' % (n, f, n, f))
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    want = {}
    for line in out.splitlines():
        n, f, v = line.split()
        want[(n, f)] = int(v)
    for n in STRUCTS:
        cls = getattr(zero, n)
        assert ctypes.sizeof(cls) == want[(n, "size")], n
        for f in fields[n]:
            assert getattr(cls, f).offset == want[(n, f)], (n, f)


def test_partition_matches_oracle(zero):
    for Nd in (1, 2, 3, 4, 7, 8, 16, 64):
        for N in list(range(0, 70)) + [1_000_003, 124_439_808, 6_476_005_376]:
            p = zero.zero_partition(N, Nd)
            assert (p.S, p.Np, p.pad) == oracle.partition(N, Nd)
            assert p.N == N and p.Nd == Nd


def test_partition_rejects(zero):
    for N, Nd in [(-1, 4), (10, 0), (10, 65)]:
        with pytest.raises(zero.ZeroError) as e:
            zero.zero_partition(N, Nd)
        assert e.value.code == -1
    assert "Nd=65" in zero.lib.zero_last_error().decode()


def test_accounting_matches_oracle(zero):
    for N, Nd, bpp, bpo in [(175e9, 64, 2, 12), (7e9, 8, 2, 4), (1e9, 1, 4, 8), (0.0, 3, 2, 12)]:
        a = zero.zero_memory_estimate(N, Nd, bpp, bpo)
        b = oracle.memory_estimate(N, Nd, bpp, bpo)
        for stage in b:
            for k in b[stage]:
                assert a[stage][k] == pytest.approx(b[stage][k], rel=1e-14, abs=0)
    for stage in range(4):
        for Nd in (1, 2, 8, 64):
            assert zero.zero_comm_volume(stage, 1e9, Nd) == pytest.approx(
                oracle.comm_volume(stage, 1e9, Nd), rel=1e-15)
    assert zero.zero_comm_volume(4, 1.0, 2) < 0 and zero.zero_comm_volume(1, 1.0, 0) < 0


def test_accounting_rejections_leave_a_message(zero):
    for args, word in [((-1.0, 4, 2, 12), "N"), ((1e9, 0, 2, 12), "Nd"),
                       ((1e9, 4, -2, 12), "bytes_per_param")]:
        zero.lib.zero_partition(-1, 4, None)  # leaves an unrelated message behind
        with pytest.raises(zero.ZeroError) as e:
            zero.zero_memory_estimate(*args)
        assert e.value.code == zero.ZERO_EINVAL and word in str(e.value), args


def test_workspace_and_version(zero):
    assert 256 < zero.zero_workspace_bytes() < (1 << 20)
    assert "sm_100a" in zero.zero_version()


def test_entry_points_validate_before_touching_the_device(zero):
    hp = zero.hparams(1e-3)
    st = zero.zero_state_t()
    cases = [
        lambda: zero.zero_step(4, 4, 10, 0, st, hp),                      # bad stage
        lambda: zero.zero_step(1, 0, 10, 0, st, hp),                      # bad Nd
        lambda: zero.zero_step(1, 4, -1, 0, st, hp),                      # bad N
        lambda: zero.zero_step(1, 4, 10, 0, st, zero.hparams(1e-3, beta1=1.0)),
        lambda: zero.zero_step(1, 4, 10, 0, st, zero.hparams(1e-3, eps=0.0)),
        lambda: zero.zero_step(1, 4, 10, 0, st, zero.hparams(1e-3, loss_scale=0.0)),
        lambda: zero.zero_step(1, 4, 10, 0, st, hp),                      # NULL workspace
        lambda: zero.zero_reduce_scatter([0] * 4, 0, 4, 0, 8, hp, 0, 0),  # NULL pointers
        lambda: zero.zero_reduce_scatter([8] * 4, 2, 4, 0, 8, hp, 16, 16),  # bad dtype
        lambda: zero.zero_reduce_scatter([16] * 4, 0, 4, 5, 4, hp, 16, 16),  # hi < lo
        lambda: zero.zero_adam_shard(0, 0, 0, 0, 0, 8, hp, None, 0),
        lambda: zero.zero_allgather(16, [16] * 2, 2, 0, 8, 7, 16),          # bad gate
        lambda: zero.zero_allgather(16, [16] * 2, 2, 0, 8, 1, None),        # gate needs ws
        lambda: zero.zero3_gather_layer([16] * 2, 2, 8, [16] * 2 * 33),     # nout too large
        lambda: zero.zero3_gather_layer([16] * 2, 2, -1, [16]),
        lambda: zero.zero_workspace_init(None, 0),
        lambda: zero.zero_workspace_init(16, -3),
        lambda: zero.zero_step(1, 4, 10, 0, st, zero.hparams(1e-3, max_grad_norm=-1.0)),
        lambda: zero.zero_loss_scaler_init(None, 1024.0),
        lambda: zero.zero_loss_scaler_init(16, 0.0),
        lambda: zero.zero_loss_scaler_init(16, 1024.0, growth_factor=0.5),
        lambda: zero.zero_loss_scaler_init(16, 1024.0, backoff_factor=1.5),
        lambda: zero.zero_loss_scaler_init(16, 1024.0, growth_interval=0),
        lambda: zero.zero_test_inject_stall(-2),
    ]
    for k, call in enumerate(cases):
        with pytest.raises(zero.ZeroError) as e:
            call()
        assert e.value.code == zero.ZERO_EINVAL, k
        assert zero.lib.zero_last_error().decode() != ""


def test_misaligned_workspace_is_refused(zero):
    """A workspace off a 16-byte boundary is refused before any device work (the kernels would
    update its doubles and 64-bit counters at misaligned addresses)."""
    hp = zero.hparams(1e-3)
    st = zero.zero_state_t()
    st.workspace = 4096 + 8  # fake, never dereferenced
    cases = [
        lambda: zero.zero_step(2, 4, 10, 0, st, hp),
        lambda: zero.zero_workspace_init(4096 + 8, 0),
        lambda: zero.zero_loss_scaler_init(4096 + 4, 1024.0),
        lambda: zero.zero_allgather(16, [16] * 2, 2, 0, 8, 1, 4096 + 8),
        lambda: zero.zero_reduce_scatter([16] * 4, 0, 4, 0, 8, hp, 16, 4096 + 8),
    ]
    for k, call in enumerate(cases):
        with pytest.raises(zero.ZeroError) as e:
            call()
        assert e.value.code == zero.ZERO_EINVAL and "16-byte aligned" in str(e.value), k


def test_fused_step_refuses_clipping(zero):
    st = zero.zero_state_t()
    st.grad_dtype = zero.ZERO_BF16
    st.flags = zero.ZERO_FUSED
    for r in range(4):  # fake, never dereferenced: the call is refused before any device work
        st.grads[r] = 4096
        st.params[r] = 4096
    st.workspace = 4096
    with pytest.raises(zero.ZeroError) as e:
        zero.zero_step(1, 4, 1000, 0, st, zero.hparams(1e-3, max_grad_norm=1.0))
    assert e.value.code == zero.ZERO_EINVAL and "ZERO_TWO_PASS" in str(e.value)
    st.flags = zero.ZERO_FUSED | zero.ZERO_BF16_GRAD_SHARD  # no gradient shard to keep
    with pytest.raises(zero.ZeroError) as e:
        zero.zero_step(2, 4, 1000, 0, st, zero.hparams(1e-3))
    assert "ZERO_BF16_GRAD_SHARD" in str(e.value)


def test_fused_layers_refusals(zero):
    """Stage 3 with ZERO_FUSED_LAYERS: clipping, a bf16 gradient shard or a missing second state
    copy are refused before any device work."""
    st = zero.zero_state_t()
    st.grad_dtype = zero.ZERO_BF16
    st.flags = zero.ZERO_FUSED_LAYERS
    for r in range(4):  # fake, never dereferenced
        st.grads[r] = 4096
        st.params[r] = 4096
    for k in range(2):
        st.master[k] = st.exp_avg[k] = st.exp_avg_sq[k] = 4096
    st.param_shard = 4096
    st.workspace = 4096
    with pytest.raises(zero.ZeroError) as e:
        zero.zero_step(3, 4, 1000, 500, st, zero.hparams(1e-3, max_grad_norm=1.0))
    assert e.value.code == zero.ZERO_EINVAL and "clip" in str(e.value)
    st.flags = zero.ZERO_FUSED_LAYERS | zero.ZERO_BF16_GRAD_SHARD
    with pytest.raises(zero.ZeroError) as e:
        zero.zero_step(3, 4, 1000, 500, st, zero.hparams(1e-3))
    assert "ZERO_BF16_GRAD_SHARD" in str(e.value)
    st.flags = zero.ZERO_FUSED_LAYERS
    st.master[1] = 0
    with pytest.raises(zero.ZeroError) as e:
        zero.zero_step(3, 4, 1000, 500, st, zero.hparams(1e-3))
    assert "both state copies" in str(e.value)


def test_offload_step_validates_before_touching_the_device(zero):
    hp = zero.hparams(1e-3)
    st = zero.zero_offload_state_t()
    cases = [(0, 10, 0, st, hp), (4, -1, 0, st, hp), (4, 10, -1, st, hp), (4, 10, 0, st, hp),
             (4, 10, 0, st, zero.hparams(1e-3, eps=-1.0))]
    for args in cases:
        with pytest.raises(zero.ZeroError) as e:
            zero.zero_offload_step(*args)
        assert e.value.code == zero.ZERO_EINVAL
    st.workspace = 4096  # fake: the missing staging buffers are refused first
    with pytest.raises(zero.ZeroError) as e:
        zero.zero_offload_step(4, 10, 0, st, hp)
    assert "grad_dev" in str(e.value)


def test_workspace_header_offsets_used_by_the_multi_gpu_path(tmp_path):
    """dist.py all-reduces the pending overflow flag and sum of squares in place in the
    workspace header by byte offset; the device header (compiled here for the host with nvcc,
    nothing runs on a GPU) has them at those offsets, fits its 256-byte slot, and is what
    zero_read_result copies."""
    from zero_sharded_optimizer_03_b200 import dist
    src = tmp_path / "hdr.cu"
    src.write_text(
        '#include <cstdio>\n#include <cstddef>\n#include "zero_kernels.cuh"\n'
        "int main() {\n"
        '  std::printf("%zu %zu %zu\\n", offsetof(zb::Header, pending_flag),\n'
        "              offsetof(zb::Header, pending_sumsq), sizeof(zb::Header));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "hdr"
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I",
                    os.path.join(ROOT, "zero_sharded_optimizer_03_b200", "csrc"), str(src),
                    "-o", str(exe)], check=True)
    flag, sumsq, size = map(int, subprocess.run([str(exe)], capture_output=True, text=True,
                                                check=True).stdout.split())
    assert (flag, sumsq) == (dist.PENDING_FLAG_OFFSET, dist.PENDING_SUMSQ_OFFSET)
    assert size <= 256
