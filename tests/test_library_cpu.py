"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every function the public header declares, the binding mirrors those names,
and the product package never reaches the oracle."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, 'include', 'llama_b200.h')
PKG = os.path.join(ROOT, 'llama_transformer_decoder_b200')


def _declared():
    src = open(HEADER).read()
    src = re.sub(r'/\*.*?\*/', '', src, flags=re.S)
    return sorted(set(re.findall(r'\b(llama_[a-z_0-9]+)\s*\(', src)))


def test_library_exports_header_symbols():
    from llama_transformer_decoder_b200 import binding
    out = subprocess.run(['nm', '-D', '--defined-only', binding.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r' T (llama_\w+)', out))
    declared = _declared()
    assert len(declared) >= 25
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    # the binding wraps each declared function under the same name
    assert sorted(binding.exported_symbols()) == declared
    for f in declared:
        assert callable(getattr(binding, f))


def test_host_only_entry_points():
    from llama_transformer_decoder_b200 import binding as b
    assert b.llama_ffn_hidden(4096, 1024, 1.3) == 14336
    assert b.llama_ffn_hidden(256, 256, 0.0) == 768
    from oracle import ffn_hidden_dim
    for dim, mo, mult in [(4096, 1024, 1.3), (2048, 256, 1.5), (512, 64, 0.0), (5120, 256, 1.3)]:
        assert b.llama_ffn_hidden(dim, mo, mult) == ffn_hidden_dim(dim, mo, mult if mult > 0 else None)
    assert b.status_string(0) == 'ok'
    assert 'timed out' in b.status_string(b.LLAMA_ERR_DEVICE_TIMEOUT)


def test_product_never_touches_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(('.py', '.cu', '.cuh', '.h', '.cpp')):
                text = open(os.path.join(dirpath, f), encoding='utf-8').read()
                assert 'import oracle' not in text and 'from oracle' not in text, f
                assert 'seeded_inputs' not in text, f


def test_sm100a_only_build_flags():
    from llama_transformer_decoder_b200 import build
    assert build.ARCH == ['-gencode', 'arch=compute_100a,code=sm_100a']


def test_binding_fails_loudly_without_library(tmp_path):
    """Importing the binding where no library was built raises ImportError."""
    dst = tmp_path / 'binding.py'
    dst.write_text(open(os.path.join(PKG, 'binding.py')).read())
    r = subprocess.run(['python', '-c', f"import importlib.util as u; s=u.spec_from_file_location('b', {str(dst)!r});"
                        "m=u.module_from_spec(s); s.loader.exec_module(m)"], capture_output=True, text=True)
    assert r.returncode != 0 and 'ImportError' in r.stderr


@pytest.mark.parametrize('over,dtype,status', [
    (dict(n_heads=7), 'F32', 'SHAPE'),                     # heads do not divide dim
    (dict(n_kv_heads=3), 'F32', 'SHAPE'),                  # kv heads do not divide heads
    (dict(dim=0), 'F32', 'SHAPE'),
    (dict(n_heads=32, n_kv_heads=2), 'F32', 'UNSUPPORTED'),  # more than 8 query heads per kv head
    (dict(dim=2048, n_heads=32, n_kv_heads=8), 'BF16', 'UNSUPPORTED'),  # 16-bit kernels need head_dim 128
    (dict(kv_page_size=64), 'BF16', 'UNSUPPORTED'),          # pages are 128 positions
    (dict(kv_page_size=128), 'F32', 'UNSUPPORTED'),          # paged kernels are 16-bit
    (dict(kv_page_size=128, kv_pages=-1), 'BF16', 'SHAPE'),
    (dict(ffn_hidden=0, multiple_of=0), 'F32', 'SHAPE'),     # no hidden size and no rule to derive it
    (dict(norm_eps=-1.0), 'F32', 'INVALID_ARG'),
    (dict(rope_theta=0.0), 'F32', 'INVALID_ARG'),
])
def test_config_validation_on_host(over, dtype, status):
    """llama_create rejects an invalid configuration before touching the
    device, with the status the header documents."""
    from llama_transformer_decoder_b200 import binding as b
    from llama_transformer_decoder_b200.configs import make_config
    base = dict(dim=4096, n_layers=1, n_heads=32, n_kv_heads=8, vocab_size=1000, ffn_hidden=14336,
                multiple_of=1024, norm_eps=1e-5, rope_theta=500000.0)
    cfg = make_config(base, dtype=getattr(b, 'LLAMA_' + dtype), max_batch=2, max_seq=256, **over)
    with pytest.raises(b.LlamaError) as e:
        b.llama_create(cfg)
    assert e.value.status == getattr(b, 'LLAMA_ERR_' + status)


def test_unknown_dtype_is_rejected_on_host():
    from llama_transformer_decoder_b200 import binding as b
    from llama_transformer_decoder_b200.configs import TINY, make_config
    with pytest.raises(b.LlamaError) as e:
        b.llama_create(make_config(TINY, dtype=7, max_batch=1, max_seq=16))
    assert e.value.status == b.LLAMA_ERR_INVALID_ARG
