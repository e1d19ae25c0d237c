"""B200 (sm_100a) paged MLA decode.

`mla_paged_kv_06_b200.mla` binds the C ABI of libmla_b200.so (include/mla.h);
`mla_paged_kv_06_b200.workloads` draws seeded synthetic inputs. Importing the package
does not load the library; importing `.mla` does, and fails if it is not built.
"""
