"""The C ABI library loads and exports every entry point that include/smdm.h declares (CPU)."""
import ctypes
import os
import re

import pytest

import masked_discrete_diffusion_sparse_b200 as smdm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "smdm.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(smdm_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("smdm_create", "smdm_prefill", "smdm_step", "smdm_generate",
              "smdm_forward_stepcausal"):
        assert s in syms


def test_library_exports_every_declared_symbol():
    if not os.path.exists(smdm.LIB_PATH):
        from masked_discrete_diffusion_sparse_b200 import build
        build.build()
    lib = smdm.lib()
    for s in declared_symbols():
        assert hasattr(lib, s), s
    assert set(declared_symbols()) <= set(smdm.EXPORTED)


def test_invalid_config_is_rejected_without_gpu():
    lib = smdm.lib()
    bad = smdm.make_config(2, 100, 3, 33, 64, 10, dtype=smdm.SMDM_BF16, max_batch=1, max_len=10,
                           max_step_rows=10, max_rows=10)
    assert lib.smdm_workspace_bytes(ctypes.byref(bad)) == 0
    bad2 = smdm.make_config(2, 256, 2, 128, 704, 1000, dtype=smdm.SMDM_BF16, max_batch=99,
                            max_len=10, max_step_rows=10, max_rows=10)
    assert lib.smdm_workspace_bytes(ctypes.byref(bad2)) == 0


def test_config_rules_for_bf16_models():
    """bf16 shape rules of the header: d_model % 128, d_head in {64, 128}, d_ffn % 64 and
    vocab % 4 (16-byte logit rows); a valid shape gets a positive workspace size."""
    lib = smdm.lib()
    ok = dict(dtype=smdm.SMDM_BF16, max_batch=1, max_len=300, max_step_rows=200, max_rows=300)
    good = smdm.make_config(2, 256, 2, 128, 704, 1000, **ok)
    assert lib.smdm_workspace_bytes(ctypes.byref(good)) > 0
    for shape in [(2, 192, 3, 64, 704, 1000),    # d_model % 128
                  (2, 256, 8, 32, 704, 1000),    # d_head 32
                  (2, 256, 2, 128, 700, 1000),   # d_ffn % 64
                  (2, 256, 2, 128, 704, 1002)]:  # vocab % 4
        bad = smdm.make_config(*shape, **ok)
        assert lib.smdm_workspace_bytes(ctypes.byref(bad)) == 0, shape
    # the length-token variant (n_reg = SMDM_REG_LEN) is a valid config; below it is not
    len_cfg = smdm.make_config(2, 256, 2, 128, 704, 1000, n_reg=smdm.SMDM_REG_LEN, **ok)
    assert lib.smdm_workspace_bytes(ctypes.byref(len_cfg)) > 0
    below = smdm.make_config(2, 256, 2, 128, 704, 1000, n_reg=-2, **ok)
    assert lib.smdm_workspace_bytes(ctypes.byref(below)) == 0
    # the fp32 path has none of the tile rules
    f32 = smdm.make_config(2, 128, 2, 64, 320, 301, dtype=smdm.SMDM_F32, max_batch=1,
                           max_len=100, max_step_rows=100, max_rows=100)
    assert lib.smdm_workspace_bytes(ctypes.byref(f32)) > 0


def test_model_refuses_to_run_without_cuda():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    cfg = smdm.make_config(2, 256, 2, 128, 704, 1000, max_batch=1, max_len=300,
                           max_step_rows=200, max_rows=300)
    with pytest.raises(RuntimeError):
        smdm.Model(cfg, {})


def test_argument_errors_return_before_any_device_work():
    """The header's error rule: argument errors are reported on the host, before any launch.
    A null handle or null weights give SMDM_EINVAL, an invalid shape SMDM_ESHAPE, with no CUDA
    call (this runs without a GPU)."""
    lib = smdm.lib()
    E = smdm.SMDM_EINVAL
    assert lib.smdm_prefill(None, 0, None, 4, 8, None, None) == E
    assert lib.smdm_prefill_given(None, 0, None, 4, 8, None, None, 0, None, None) == E
    assert lib.smdm_step(None, 1, None, None, None, None, None) == E
    assert lib.smdm_step_switched(None, None, 7, None, None, None, None) == E
    assert lib.smdm_dense_step(None, None, None, None, None, None) == E
    assert lib.smdm_generate(None, 1, None, 4, 8, None, 0, None, None) == E
    assert lib.smdm_forward_stepcausal(None, None, None, None, None, 1, None, 1, None, None) == E
    assert lib.smdm_debug_mask(None, None, None, 1, None, None) == E
    n = ctypes.c_int(0)
    assert lib.smdm_debug_rows(None, None, None, None, None, ctypes.byref(n), None) == E
    assert lib.smdm_profile_begin(None, 1) == E
    assert lib.smdm_profile_end(None, None, None) == E
    bits = ctypes.c_uint(0)
    assert lib.smdm_device_status(None, ctypes.byref(bits), None) == E
    assert lib.smdm_context_length(None, 0) == -1
    assert lib.smdm_last_error(None) == b"null handle"
    lib.smdm_destroy(None)

    good = smdm.make_config(2, 256, 2, 128, 704, 1000, dtype=smdm.SMDM_BF16, max_batch=1,
                            max_len=300, max_step_rows=200, max_rows=300)
    bad = smdm.make_config(2, 192, 3, 64, 704, 1000, dtype=smdm.SMDM_BF16, max_batch=1,
                           max_len=300, max_step_rows=200, max_rows=300)
    out = ctypes.c_void_p(1)
    assert lib.smdm_create(ctypes.byref(bad), None, None, 0, ctypes.byref(out)) == \
        smdm.SMDM_ESHAPE
    assert out.value is None                       # *out is cleared on every failure
    assert lib.smdm_create(ctypes.byref(good), None, None, 0, ctypes.byref(out)) == E
    assert lib.smdm_create(ctypes.byref(good), None, None, 0, None) == E
    w = smdm.smdm_weights()                        # every pointer null
    assert lib.smdm_forward_stepcausal_noalloc(ctypes.byref(good), ctypes.byref(w), None, None,
                                               None, None, 4, None, 1, None, None) == E
    assert lib.smdm_forward_stepcausal_noalloc(ctypes.byref(bad), ctypes.byref(w), None, None,
                                               None, None, 4, None, 1, None, None) == \
        smdm.SMDM_ESHAPE
    # one layer's norm gain missing: refused on the host, before any CUDA call (the pointers
    # below are never dereferenced)
    fake = ctypes.c_void_p(0x1000)
    nl = good.n_layers
    per_layer = {k: (ctypes.c_void_p * nl)(*([fake.value] * nl))
                 for k in ("attn_norm", "w_qkv", "w_o", "mlp_norm", "w_gate", "w_up", "w_down")}
    per_layer["mlp_norm"][nl - 1] = None
    w2 = smdm.smdm_weights(fake, fake, fake, *[ctypes.cast(per_layer[k], smdm._PP) for k in
                                              ("attn_norm", "w_qkv", "w_o", "mlp_norm",
                                               "w_gate", "w_up", "w_down")])
    assert lib.smdm_forward_stepcausal_noalloc(ctypes.byref(good), ctypes.byref(w2), fake, fake,
                                               fake, fake, 4, fake, 1, fake, None) == E


def test_capacities_that_overflow_32_bit_indices_are_rejected():
    lib = smdm.lib()
    base = dict(dtype=smdm.SMDM_BF16, max_batch=1, max_step_rows=200, max_rows=300)
    ok = smdm.make_config(2, 256, 2, 128, 704, 1000, max_len=300, **base)
    assert lib.smdm_workspace_bytes(ctypes.byref(ok)) > 0
    huge = smdm.make_config(2, 256, 2, 128, 704, 1000, max_len=(1 << 30), **base)
    assert lib.smdm_workspace_bytes(ctypes.byref(huge)) == 0
    regs = smdm.make_config(2, 256, 2, 128, 704, 1000, n_reg=(1 << 17), max_len=300, **base)
    assert lib.smdm_workspace_bytes(ctypes.byref(regs)) == 0


def test_binding_struct_layouts_match_the_header(tmp_path):
    """Every ABI struct of the Python binding has the size and field offsets that a C compiler
    gives the header's struct (a program compiled here against include/smdm.h prints them)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    structs = {"smdm_config": smdm.smdm_config, "smdm_weights": smdm.smdm_weights,
               "smdm_step_desc": smdm.smdm_step_desc, "smdm_plan": smdm.smdm_plan,
               "smdm_profile": smdm.smdm_profile}
    lines = ['#include <stdio.h>', '#include "smdm.h"', "int main(void) {"]
    for name, cls in structs.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for f in cls._fields_:
            lines.append(f'  printf("{name} {f[0]} %zu\\n", offsetof({name}, {f[0]}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src), "-o",
                    str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True,
                               text=True).stdout.splitlines():
        name, field, value = line.split()
        got[(name, field)] = int(value)
    for name, cls in structs.items():
        assert got[(name, "size")] == ctypes.sizeof(cls), name
        for f in cls._fields_:
            assert got[(name, f[0])] == getattr(cls, f[0]).offset, (name, f[0])


def test_plain_c_program_links_and_calls_the_library(tmp_path):
    """The boundary is usable from C: a C program compiled against include/smdm.h and linked
    with libsmdm.so sizes a workspace and gets the host-side errors (no GPU needed)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    if not os.path.exists(smdm.LIB_PATH):
        from masked_discrete_diffusion_sparse_b200 import build
        build.build()
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    src = tmp_path / "use.c"
    src.write_text(r'''
#include <stdio.h>
#include "smdm.h"
int main(void) {
  smdm_config c = {0};
  c.n_layers = 2; c.d_model = 256; c.n_heads = 2; c.d_head = 128; c.d_ffn = 704;
  c.vocab = 1000; c.n_reg = 64; c.dtype = SMDM_BF16; c.rope_theta = 10000.f; c.rms_eps = 1e-6f;
  c.max_batch = 1; c.max_len = 300; c.max_step_rows = 200; c.max_rows = 300;
  size_t ws = smdm_workspace_bytes(&c);
  smdm_handle* h = (smdm_handle*)1;
  int s1 = smdm_create(&c, NULL, NULL, ws, &h);
  int s2 = smdm_step(NULL, 1, NULL, NULL, NULL, NULL, 0);
  c.d_model = 192;
  size_t bad = smdm_workspace_bytes(&c);
  printf("%zu %d %d %d %zu %s\n", ws, s1, h == NULL, s2, bad, smdm_last_error(NULL));
  return 0;
}
''')
    exe = tmp_path / "use"
    libdir = os.path.dirname(smdm.LIB_PATH)
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lsmdm",
                    "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert int(out[0]) > 0
    assert int(out[1]) == smdm.SMDM_EINVAL and out[2] == "1"
    assert int(out[3]) == smdm.SMDM_EINVAL
    assert int(out[4]) == 0
    assert " ".join(out[5:]) == "null handle"
