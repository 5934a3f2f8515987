"""Host-side helpers of bench.py that need no GPU."""
import bench


def test_strip_c_comments_keeps_code_and_strings():
    src = ('int a; // line comment\n/* block\n comment */ const char *s = '
           '"x // not a comment /* nor this */";\n  int   b;\n')
    assert bench.strip_c_comments(src) == (
        'int a; const char *s = "x // not a comment /* nor this */"; int b;')


def test_source_digest_ignores_comments_only():
    a = "asm(\"add.rn.f32x2 %0, %1, %2;\"); // the sum\nint x = 1;"
    b = "/* reworded */ asm(\"add.rn.f32x2 %0, %1, %2;\");\nint x = 1; // another"
    c = "asm(\"add.rn.f32x2 %0, %1, %2;\");\nint x = 2;"
    assert bench.strip_c_comments(a) == bench.strip_c_comments(b)
    assert bench.strip_c_comments(a) != bench.strip_c_comments(c)
