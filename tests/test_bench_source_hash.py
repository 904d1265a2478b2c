"""The DRAM-traffic tag in bench.py: a hash of the kernel sources that a
comment or whitespace edit leaves unchanged and a code edit changes."""

import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_for_hash", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_comments_and_whitespace_do_not_count():
    b = _bench()
    src = 'int f(int x) {\n    return x + 1;   // add one\n}\n/* block\n comment */ int g;\n'
    edited = 'int f(int x)\n{ return x + 1; // increment\n}\nint g; /* other */\n'
    assert b._code_only(src) == b._code_only(edited)


def test_code_and_string_edits_count():
    b = _bench()
    a = 'asm("tcgen05.commit // not a comment"); int x = 1;'
    # text inside a string literal is kept (whitespace is dropped everywhere)
    assert "tcgen05.commit//notacomment" in b._code_only(a)
    assert b._code_only(a) != b._code_only(a.replace("x = 1", "x = 2"))
    assert b._code_only('int y = 1;') != b._code_only('int y = 1 ;int z;')


def test_hash_covers_the_kernel_sources():
    b = _bench()
    h = b.kernel_source_hash()
    assert isinstance(h, str) and len(h) == 16
    assert h == b.kernel_source_hash()
