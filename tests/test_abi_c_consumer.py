"""The boundary used from C: tests/cpp/abi_consumer.c includes both public
headers as C99 (gcc, -pedantic -Werror), links libllama_b200.so and calls the
host-side entry points.  Its sizes must equal what the Python binding reads
through ctypes and what the Admin Guide's formulas give (the SwiGLU width of
§8.4, the KV-cache footprint of §6.2); its argument errors must come back as
the documented status codes with a message naming the fault; and nothing it calls launches a
kernel.  No GPU is needed."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

llb = pytest.importorskip("decoder_only_transformer_llama_b200",
                          reason="library not built (run decoder_only_transformer_llama_b200/build.py)")
from oracle import llama_oracle as O  # noqa: E402

# the shapes abi_consumer.c sizes: (dim, layers, heads, kv heads, vocab, multiple_of, multiplier, S, B, dtype)
SHAPES = {
    "7b": (4096, 32, 32, 32, 32000, 256, None, 4096, 4, "bf16"),
    "13b": (5120, 40, 40, 40, 32000, 256, None, 1152, 16, "f16"),
    "70b_slice": (8192, 16, 64, 8, 32000, 4096, 1.3, 4096, 8, "bf16"),
    "tiny": (256, 2, 8, 2, 512, 256, None, 128, 2, "f32"),
}


@pytest.fixture(scope="module")
def records():
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(llb.LIB_PATH)
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "abi_consumer")
        r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                            "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "cpp", "abi_consumer.c"),
                            "-o", exe, "-L", lib_dir, "-l:" + os.path.basename(llb.LIB_PATH),
                            "-Wl,-rpath," + lib_dir],
                           capture_output=True, text=True, timeout=300)
        assert r.returncode == 0, r.stderr[-4000:]
        out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = out.stdout.strip().splitlines()
    assert lines[-1] == "done"
    recs = {}
    for ln in lines[:-1]:
        f = ln.split(maxsplit=3) if ln.startswith("check ") else ln.split()
        if f[0] in ("bytes", "check"):
            recs[(f[0], f[1])] = f[2:]
        else:
            recs[f[0]] = f[1:]
    return recs


def test_struct_sizes_seen_from_c(records):
    import ctypes
    n_args, n_sampling = map(int, records["sizes"])
    assert n_args == ctypes.sizeof(llb.ModelArgs) == 13 * 4
    assert n_sampling == ctypes.sizeof(llb.Sampling) == 8


@pytest.mark.parametrize("name", list(SHAPES))
def test_sizes_from_c_match_binding_and_formulas(records, name):
    dim, L, nh, nkv, V, mo, mult, S, B, dt = SHAPES[name]
    rc, w, kv, ws, total, hidden = map(int, records[("bytes", name)])
    assert rc == llb.LLAMA_OK
    py = llb.model_bytes(llb.make_args(dim, L, nh, nkv, V, mo, mult, max_seq_len=S, max_batch_size=B, dtype=dt))
    assert (w, kv, ws, total, hidden) == (py["weights"], py["kv"], py["workspace"], py["total"], py["hidden"])
    assert hidden == O.ffn_hidden_dim(dim, mo, mult)
    esz = 4 if dt == "f32" else 2
    per_tensor = O.kv_cache_bytes_per_tensor(B, S, nkv, dim // nh, esz)
    assert 2 * L * per_tensor <= kv <= 2 * L * per_tensor + 512
    assert total == w + kv + ws


def test_sizes_of_the_published_widths(records):
    # SwiGLU widths of the 7B, 13B and 70B models (Admin Guide §8.4 rule)
    assert int(records[("bytes", "7b")][-1]) == 11008
    assert int(records[("bytes", "13b")][-1]) == 13824
    assert int(records[("bytes", "70b_slice")][-1]) == 28672


@pytest.mark.parametrize("what,code,word", [
    ("kv_heads_not_dividing", "LLAMA_ERR_INVALID_ARG", "n_kv_heads"),
    ("unknown_dtype", "LLAMA_ERR_INVALID_ARG", "dtype"),
    ("null_args", "LLAMA_ERR_INVALID_ARG", "NULL"),
    ("create_null_arena", "LLAMA_ERR_INVALID_ARG", "arena"),
    ("create_left_null", "LLAMA_OK", None),
    ("prefill_null_model", "LLAMA_ERR_INVALID_ARG", "tokens"),
    ("decode_null_model", "LLAMA_ERR_INVALID_ARG", "pos"),
    ("sample_no_uniforms", "LLAMA_ERR_INVALID_ARG", "uniforms"),
    ("logprobs_empty", "LLAMA_OK", None),
    ("op_linear_bad_dtype", "LLAMA_ERR_INVALID_ARG", "dtype"),
    ("status_null_model", "LLAMA_ERR_INVALID_ARG", "device_status"),
])
def test_status_codes_seen_from_c(records, what, code, word):
    """Each error comes back with its status code and a message that names
    what was wrong (each call's message replaces the one before it)."""
    rec = records[("check", what)]
    assert int(rec[0]) == getattr(llb, code)
    if word is not None:
        assert len(rec) == 2 and word in rec[1], rec


def test_host_calls_launch_nothing(records):
    assert int(records["launches"][0]) == 0
