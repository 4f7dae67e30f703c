"""B200-native paged KV-cache decode path.

``pagedattn`` binds the C-ABI library ``libpagedattn.so`` (CUDA kernels for
sm_100a); ``workload`` builds seeded synthetic inputs.  Importing the package
loads nothing: the library is opened on first use of ``pagedattn``.
"""
