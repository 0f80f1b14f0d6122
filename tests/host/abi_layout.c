/* Prints the size and field offsets of the C ABI's segment structs, as the
 * C compiler lays them out, for tests/test_host_units.py to compare with the
 * ctypes binding. */
#include <stddef.h>
#include <stdio.h>

#include "ds.h"

#define F(T, f) printf(#T " " #f " %zu\n", offsetof(T, f))

int main(void)
{
    printf("ds_wseg size %zu\n", sizeof(ds_wseg));
    F(ds_wseg, w); F(ds_wseg, gain); F(ds_wseg, w_eff); F(ds_wseg, gy); F(ds_wseg, grad_w); F(ds_wseg, grad_g);
    F(ds_wseg, rows); F(ds_wseg, cols); F(ds_wseg, ld); F(ds_wseg, ld_out); F(ds_wseg, radius);
    F(ds_wseg, gain_scalar); F(ds_wseg, rnorm); F(ds_wseg, transposed); F(ds_wseg, tgroup);
    printf("ds_aseg size %zu\n", sizeof(ds_aseg));
    F(ds_aseg, x); F(ds_aseg, r); F(ds_aseg, y); F(ds_aseg, alpha); F(ds_aseg, rows); F(ds_aseg, cols);
    F(ds_aseg, ld);
    return 0;
}
