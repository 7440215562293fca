"""The C-ABI library builds, loads and exports what include/wedlm.h declares
(no GPU needed: nothing here launches a kernel)."""
import ctypes
import os
import subprocess

import pytest

from streaming_decoding_b200 import _lib
from streaming_decoding_b200._lib import ModelCfg, SeqStats, StepParams

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_library_exports_every_declared_function():
    lib = _lib.load()
    names = _lib.header_functions()
    assert len(names) >= 15
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # and the binding declares a signature for each of them
    assert sorted(_lib._SIGS) == names


def test_exported_symbols_are_unmangled_c():
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in _lib.header_functions():
        assert n in exported, n


def _c_layout(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(r'''
#include <stdio.h>
#include <stddef.h>
#include "wedlm.h"
#define P(T, f) printf(#T "." #f " %zu\n", offsetof(T, f))
int main(void) {
  printf("sizeof.cfg %zu\nsizeof.params %zu\nsizeof.stats %zu\n", sizeof(wedlm_model_cfg),
         sizeof(wedlm_step_params), sizeof(wedlm_seq_stats));
  P(wedlm_model_cfg, rope_theta); P(wedlm_model_cfg, rms_eps); P(wedlm_model_cfg, dtype);
  P(wedlm_model_cfg, prefill_chunk); P(wedlm_step_params, tau_none); P(wedlm_step_params, logit_scale);
  P(wedlm_step_params, blockwise); P(wedlm_step_params, temperature); P(wedlm_step_params, seed);
  P(wedlm_seq_stats, committed_len); P(wedlm_seq_stats, active);
  return 0;
}
''')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    return dict(line.split() for line in subprocess.check_output([str(exe)], text=True).splitlines())


def test_struct_layouts_match_c(tmp_path):
    c = _c_layout(tmp_path)
    assert int(c["sizeof.cfg"]) == ctypes.sizeof(ModelCfg)
    assert int(c["sizeof.params"]) == ctypes.sizeof(StepParams)
    assert int(c["sizeof.stats"]) == ctypes.sizeof(SeqStats)
    assert int(c["wedlm_model_cfg.rope_theta"]) == ModelCfg.rope_theta.offset
    assert int(c["wedlm_model_cfg.rms_eps"]) == ModelCfg.rms_eps.offset
    assert int(c["wedlm_model_cfg.dtype"]) == ModelCfg.dtype.offset
    assert int(c["wedlm_model_cfg.prefill_chunk"]) == ModelCfg.prefill_chunk.offset
    assert int(c["wedlm_step_params.tau_none"]) == StepParams.tau_none.offset
    assert int(c["wedlm_step_params.logit_scale"]) == StepParams.logit_scale.offset
    assert int(c["wedlm_step_params.blockwise"]) == StepParams.blockwise.offset
    assert int(c["wedlm_step_params.temperature"]) == StepParams.temperature.offset
    assert int(c["wedlm_step_params.seed"]) == StepParams.seed.offset
    assert int(c["wedlm_seq_stats.committed_len"]) == SeqStats.committed_len.offset
    assert int(c["wedlm_seq_stats.active"]) == SeqStats.active.offset


def test_status_strings_and_constants():
    lib = _lib.load()
    C = _lib.header_constants()
    assert C["WEDLM_PAGE_TOKENS"] == 16
    for name in ("OK", "ERR_INVALID_ARG", "ERR_OOM_PAGES", "ERR_OOM_DEVICE", "ERR_CUDA", "ERR_DEVICE_ASSERT",
                 "ERR_STATE", "ERR_UNSUPPORTED", "ERR_TIMEOUT"):
        s = lib.wedlm_status_str(C["WEDLM_" + name]).decode()
        assert s and s != "unknown status"


def _cfg(**kw):
    base = dict(n_layers=2, d_model=128, n_heads=4, n_kv_heads=2, head_dim=32, ffn_dim=384, vocab=512, mask_id=511,
                rope_theta=1e4, rms_eps=1e-6, dtype=0, max_batch=1, max_window=4, max_ctx=64, num_pages=0,
                prefill_chunk=0)
    base.update(kw)
    return ModelCfg(**base)


@pytest.mark.parametrize("bad", [dict(n_heads=3), dict(mask_id=512), dict(max_window=65), dict(head_dim=33),
                                 dict(dtype=7), dict(dtype=1, head_dim=64), dict(max_batch=0), dict(vocab=1)])
def test_create_rejects_invalid_config_without_touching_the_gpu(bad):
    lib = _lib.load()
    h = ctypes.c_void_p()
    st = lib.wedlm_create(ctypes.byref(_cfg(**bad)), None, ctypes.byref(h))
    assert st == _lib.header_constants()["WEDLM_ERR_INVALID_ARG"]
    assert not h.value


def test_null_arguments_are_rejected():
    lib = _lib.load()
    C = _lib.header_constants()
    assert lib.wedlm_create(None, None, None) == C["WEDLM_ERR_INVALID_ARG"]
    assert lib.wedlm_prefill(None, 0, None, 0, 1, 1) == C["WEDLM_ERR_INVALID_ARG"]
    assert lib.wedlm_stream_step(None, None, None, None, None) == C["WEDLM_ERR_INVALID_ARG"]
    assert lib.wedlm_reorder_window(None, None, None, 1, 0, None, None, None, None, None) == C["WEDLM_ERR_INVALID_ARG"]
    assert lib.wedlm_linear_bf16(None, None, None, 16, 16, 7, None) == C["WEDLM_ERR_INVALID_ARG"]
    lib.wedlm_destroy(None)
    assert lib.wedlm_last_error(None) == b""



def test_every_declaration_is_documented():
    """Each function the header declares is preceded by a doc comment, its own
    or that of the group of declarations it closes (argument meaning, layout,
    ownership and errors live there)."""
    import re
    lines = open(os.path.join(ROOT, "include", "wedlm.h")).read().split("\n")
    decl = re.compile(r"^[A-Za-z_][\w\s\*]*?\b(wedlm_\w+)\s*\(")
    undocumented = []
    for i, line in enumerate(lines):
        m = decl.match(line)
        if not m or line.startswith(("typedef", "#")):
            continue
        j = i - 1
        while j >= 0 and (not lines[j].strip() or lines[j].startswith("#define")):
            j -= 1
        # a declaration right after another one shares that one's comment
        if not (lines[j].rstrip().endswith("*/") or lines[j].rstrip().endswith(");")):
            undocumented.append(m.group(1))
    assert not undocumented, undocumented
