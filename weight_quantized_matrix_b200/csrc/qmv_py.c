/*
 * qmv_py.c -- CPython extension "_qmv_fast": the per-call entry points of
 * libqmv.so for Python callers, with arguments passed as plain Python ints
 * (device pointers, sizes, enum values, the cudaStream_t).  It only converts
 * arguments and forwards to the C ABI of include/qmv.h; the status code is
 * returned unchanged.  Exists because ctypes argument conversion costs more
 * host time per call than a decode-size qmv takes on the GPU.
 */
#define PY_SSIZE_T_CLEAN
#include <Python.h>

#include <limits.h>

#include "qmv.h"

static int as_ptr(PyObject* o, void** out) {
    if (o == Py_None) { *out = NULL; return 0; }
    *out = PyLong_AsVoidPtr(o);
    return (*out == NULL && PyErr_Occurred()) ? -1 : 0;
}

/* A Python int that fits a C int; anything larger raises OverflowError
 * instead of being narrowed. */
static int as_int(PyObject* o, int* out) {
    long v = PyLong_AsLong(o);
    if (v == -1 && PyErr_Occurred()) return -1;
    if (v < INT_MIN || v > INT_MAX) {
        PyErr_SetString(PyExc_OverflowError, "argument does not fit a C int");
        return -1;
    }
    *out = (int)v;
    return 0;
}

/* affine(x, w, scales, biases, y, M, N, K, bits, group, dtype, batch, x_batched, stream) -> status */
static PyObject* py_affine(PyObject* self, PyObject* const* a, Py_ssize_t n) {
    (void)self;
    if (n != 14) { PyErr_SetString(PyExc_TypeError, "affine() takes 14 arguments"); return NULL; }
    void* p[5];
    int v[8];
    void* st;
    for (int i = 0; i < 5; ++i) if (as_ptr(a[i], &p[i])) return NULL;
    for (int i = 0; i < 8; ++i) if (as_int(a[5 + i], &v[i])) return NULL;
    if (as_ptr(a[13], &st)) return NULL;
    int r;
    Py_BEGIN_ALLOW_THREADS
    r = qmv_affine_batched(p[0], p[1], p[2], p[3], p[4], v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7], st);
    Py_END_ALLOW_THREADS
    return PyLong_FromLong(r);
}

/* fp(x, w, scales, global_scale, y, M, N, K, mode, dtype, batch, x_batched, stream) -> status */
static PyObject* py_fp(PyObject* self, PyObject* const* a, Py_ssize_t n) {
    (void)self;
    if (n != 13) { PyErr_SetString(PyExc_TypeError, "fp() takes 13 arguments"); return NULL; }
    void* p[5];
    int v[7];
    void* st;
    for (int i = 0; i < 5; ++i) if (as_ptr(a[i], &p[i])) return NULL;
    for (int i = 0; i < 7; ++i) if (as_int(a[5 + i], &v[i])) return NULL;
    if (as_ptr(a[12], &st)) return NULL;
    int r;
    Py_BEGIN_ALLOW_THREADS
    r = qmv_fp_batched(p[0], p[1], p[2], (const float*)p[3], p[4], v[0], v[1], v[2], v[3], v[4], v[5], v[6], st);
    Py_END_ALLOW_THREADS
    return PyLong_FromLong(r);
}

/* block_scaled(x, w, scales, global_scale, y, M, N, K, format, dtype, batch, x_batched, stream) -> status */
static PyObject* py_block_scaled(PyObject* self, PyObject* const* a, Py_ssize_t n) {
    (void)self;
    if (n != 13) { PyErr_SetString(PyExc_TypeError, "block_scaled() takes 13 arguments"); return NULL; }
    void* p[5];
    int v[7];
    void* st;
    for (int i = 0; i < 5; ++i) if (as_ptr(a[i], &p[i])) return NULL;
    for (int i = 0; i < 7; ++i) if (as_int(a[5 + i], &v[i])) return NULL;
    if (as_ptr(a[12], &st)) return NULL;
    int r;
    Py_BEGIN_ALLOW_THREADS
    r = qmv_block_scaled_batched(p[0], p[1], p[2], (const float*)p[3], p[4], v[0], v[1], v[2], v[3], v[4], v[5],
                                 v[6], st);
    Py_END_ALLOW_THREADS
    return PyLong_FromLong(r);
}

static PyMethodDef methods[] = {
    {"affine", (PyCFunction)(void (*)(void))py_affine, METH_FASTCALL, "qmv_affine_batched"},
    {"fp", (PyCFunction)(void (*)(void))py_fp, METH_FASTCALL, "qmv_fp_batched"},
    {"block_scaled", (PyCFunction)(void (*)(void))py_block_scaled, METH_FASTCALL, "qmv_block_scaled_batched"},
    {NULL, NULL, 0, NULL},
};

static struct PyModuleDef module = {PyModuleDef_HEAD_INIT, "_qmv_fast", NULL, -1, methods};

PyMODINIT_FUNC PyInit__qmv_fast(void) { return PyModule_Create(&module); }
