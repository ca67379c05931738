"""bench.py's fingerprint of the attention kernels' sources, which decides whether the committed ncu
DRAM traffic still describes the code: comments and blank lines must not change it, code must."""
import bench

SRC = '''#include "x.h"
// a line comment
int f(int a) {  /* a block
                   comment */
  const char* s = "not // a comment";
  char c = '/';
  return a + 1;   // trailing

}
'''


def test_strip_comments_keeps_code_and_literals():
    out = bench.strip_comments(SRC)
    assert "a line comment" not in out and "block" not in out and "trailing" not in out
    assert '"not // a comment"' in out and "'/'" in out
    assert out.splitlines() == ['#include "x.h"', "int f(int a) {", '  const char* s = "not // a comment";',
                                "  char c = '/';", "  return a + 1;", "}"]


def test_hash_ignores_comments_not_code():
    base = {name: SRC for name in bench.KERNEL_SOURCES}
    h0 = bench.kernel_source_hash(base.__getitem__)
    commented = {name: SRC.replace("// a line comment", "// reworded\n\n// more") for name in base}
    assert bench.kernel_source_hash(commented.__getitem__) == h0
    changed = {name: SRC.replace("a + 1", "a + 2") for name in base}
    assert bench.kernel_source_hash(changed.__getitem__) != h0

